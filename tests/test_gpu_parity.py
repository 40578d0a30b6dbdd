"""GPU parity: libaq (through the C ABI) against the CPU oracle, element by element.

Inputs are seeded synthetic draws from group_wise_affine_qmv_b200.inputs; every
quantized weight fed to a contraction is produced by the ORACLE quantizer, so
no oracle input comes from the CUDA path.  Bars:
* packing and codes: bit-exact; stored scales/biases: equal values;
* contractions: per-row max|y-ref|/max|ref| <= 4e-3 for half outputs, every
  row of every batch element (transformers issue #47331 probe metric);
* running-sum stress: the exact bias*sum(x) value within 1e-6 relative in fp32
  (mlx PR #4516).
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_qmv_b200 import aq, inputs
from tests.parity import (assert_rows_close, dtype_name, half_bits, oracle_linear_view, row_errors,
                          to_device_quant)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _q(w: torch.Tensor, group: int, bits: int, sdtype: str = "bf16"):
    Q = oracle.quantize(w.float().numpy(), group, bits, sdtype)
    tdt = torch.bfloat16 if sdtype == "bf16" else torch.float16
    return Q, to_device_quant(Q, DEV, tdt)


# ---------------------------------------------------------------------------
# quantize / dequantize
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("sdtype", ["bf16", "f16"])
def test_quantize_bit_exact(bits, group, sdtype):
    w = inputs.normal((67, 512), 1.0, seed=bits * 100 + group)
    w[3, :group] = 0.25  # one constant group
    Q = oracle.quantize(w.numpy(), group, bits, sdtype)
    tdt = torch.bfloat16 if sdtype == "bf16" else torch.float16
    wq, sc, bi = aq.aq_quantize(w.to(DEV), group, bits, scale_dtype=tdt)
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), Q.packed)
    assert np.array_equal(sc.float().cpu().numpy(), oracle.half_to_double(Q.scale_bits, sdtype).astype(np.float32))
    assert np.array_equal(bi.float().cpu().numpy(), oracle.half_to_double(Q.bias_bits, sdtype).astype(np.float32))


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_quantize_ties_bit_exact(bits, group):
    """Values exactly halfway between two codes (scale a power of two, (w - bias)/scale = k + 1/2
    with no rounding) take the oracle's codes, which a CPU pin fixes to the even neighbour."""
    maxq = (1 << bits) - 1
    rows = []
    for r, (s, b) in enumerate([(1.0, 0.0), (0.5, -3.0), (2.0, 5.25), (0.125, -0.5)]):
        ks = [(r * 7 + j) % maxq for j in range(group - 2)]
        g = [b, b + s * maxq] + [b + s * (k + 0.5) for k in ks]
        rows.append(g * 4)
    w = torch.tensor(rows, dtype=torch.float32)
    Q = oracle.quantize(w.numpy(), group, bits, "bf16")
    wq, sc, bi = aq.aq_quantize(w.to(DEV), group, bits, scale_dtype=torch.bfloat16)
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), Q.packed)
    assert np.array_equal(sc.float().cpu().numpy(), oracle.half_to_double(Q.scale_bits, "bf16").astype(np.float32))


@pytest.mark.parametrize("wdtype", [torch.bfloat16, torch.float16])
def test_quantize_half_input(wdtype):
    w = inputs.normal((40, 256), 0.02, dtype=wdtype, seed=9)
    Q = oracle.quantize(w.float().numpy(), 64, 4, "bf16")
    wq, sc, bi = aq.aq_quantize(w.to(DEV), 64, 4, scale_dtype=torch.bfloat16)
    assert np.array_equal(wq.cpu().numpy().view(np.uint32), Q.packed)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_dequantize_matches_oracle(bits):
    w = inputs.normal((33, 384), 1.0, seed=bits)
    Q, (wq, sc, bi) = _q(w, 32, bits)
    out = aq.aq_dequantize(wq, sc, bi, 32, bits, torch.float32).cpu().double().numpy()
    ref = Q.dequant()
    # one fp32 fma rounding
    assert np.all(np.abs(out - ref) <= 2.0 ** -23 * np.abs(ref) + 1e-30)


# ---------------------------------------------------------------------------
# probe (issue #47331): [2,K], [2,1,K], [2,4,K] -- every row of every batch element
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("entry", ["aq_qmm_t", "aq_qmv"])
def test_probe_every_row(entry):
    w, xs = inputs.probe_case()
    Q, (wq, sc, bi) = _q(w, 64, 4)
    wd = Q.dequant()
    fn = getattr(aq, entry)
    for x in xs:
        y = fn(x.to(DEV), wq, sc, bi, 64, 4)
        ref = oracle_linear_view(x, wd)
        err = row_errors(y, ref)
        assert err.size == x.numel() // x.shape[-1]
        assert np.all(err <= 4e-3), (tuple(x.shape), err)


def test_probe_batched_equals_flat_bitwise():
    """[B,1,K] and [2,4,K] give exactly the bits of the flattened 2D call."""
    w, _ = inputs.probe_case()
    _, (wq, sc, bi) = _q(w, 64, 4)
    x = inputs.normal((8, 2048), 1.0, torch.bfloat16, seed=17).to(DEV)
    flat = aq.aq_qmm_t(x, wq, sc, bi, 64, 4)
    for shape in [(8, 1, 2048), (2, 4, 2048), (1, 8, 2048)]:
        y = aq.aq_qmm_t(x.view(shape), wq, sc, bi, 64, 4)
        assert torch.equal(y.reshape(8, -1), flat), shape


# ---------------------------------------------------------------------------
# ragged-output qmv and the stress case (config: bits 2/3/5/6, G 32/128, K 4096)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", inputs.RAGGED_BITS)
@pytest.mark.parametrize("group", inputs.RAGGED_GROUPS)
@pytest.mark.parametrize("N", inputs.RAGGED_N)
def test_ragged_qmv(bits, group, N):
    for xi, x_shape in enumerate(inputs.RAGGED_X_SHAPES):
        w, x = inputs.ragged_case(bits, group, N, x_shape, seed=bits * 7 + group + N + 1000 * xi)
        Q, (wq, sc, bi) = _q(w, group, bits)
        wd = Q.dequant()
        y = aq.aq_qmm_t(x.to(DEV), wq, sc, bi, group, bits)
        ref = oracle_linear_view(x, wd)
        assert_rows_close(y, ref, x, wd)


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("group", [32, 128])
@pytest.mark.parametrize("rows", [1, 4])
def test_running_sum_stress_exact(xdtype, bits, group, rows):
    """Constant groups (scale 0, q 0, bias 1): y = sum(x) exactly, in fp32 output."""
    K = 4096
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    for N in inputs.RAGGED_N:
        Q, (wq, sc, bi) = _q(inputs.stress_w(N, K), group, bits, sd)
        assert np.all(Q.codes == 0)
        x = inputs.stress_x(K, rows, xdtype).to(DEV)
        y = aq.aq_qmm_t(x.view(rows, 1, K) if rows > 1 else x, wq, sc, bi, group, bits, out_dtype=torch.float32)
        small = 2.0 ** -9 if xdtype == torch.bfloat16 else 2.0 ** -12
        exact = (K // 2) * (1.0 + small)
        got = y.double().cpu().numpy()
        assert np.all(np.abs(got - exact) <= 1e-6 * exact), (N, got.ravel()[:4], exact)


# The same exact-sum case through every kernel of aq_qmm_t, with the kernel asserted: the
# warp-level kernel (8 and 32 rows), the tcgen05 small-M kernel (40 rows) and the tcgen05 prefill
# kernel (128 rows).  Each forms sum(x) per group with its own code; each must give the exact
# bias * sum(x) ("mlx PR #4516": exact result for inputs whose running sum is not representable in
# half types).  Every bits x group the kernel takes; N over the ragged set.
_WARP_BG = [(2, 64), (2, 128), (4, 32), (4, 64), (4, 128), (8, 32), (8, 64), (8, 128)]
_STRESS_KERNELS = {
    "warp_m8": (8, 4096, "warp_mma", _WARP_BG, (1, 4, 7, 1001, 4099)),
    "warp_m32": (32, 1024, "warp_mma", _WARP_BG, (1, 4, 7, 1001, 1024)),
    "tc_small_m": (40, 4096, "tc_small_m", [(b, g) for b in (2, 4, 6, 8) for g in (32, 64, 128)],
                   (1, 7, 1001, 4099)),
    "tc_prefill": (128, 4096, "tc_prefill", [(b, g) for b in (2, 4, 6, 8) for g in (64, 128)],
                   (1, 7, 1001, 4099)),
}


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", list(_STRESS_KERNELS))
def test_running_sum_stress_every_kernel(xdtype, case):
    rows, K, kernel, bgs, Ns = _STRESS_KERNELS[case]
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    small = 2.0 ** -9 if xdtype == torch.bfloat16 else 2.0 ** -12
    exact = (K // 2) * (1.0 + small)
    x = inputs.stress_x(K, rows, xdtype).to(DEV).view(rows, 1, K)
    for bits, group in bgs:
        for N in Ns:
            Q, (wq, sc, bi) = _q(inputs.stress_w(N, K), group, bits, sd)
            assert np.all(Q.codes == 0)
            y = torch.empty(rows, 1, N, dtype=torch.float32, device=DEV)
            assert aq.aq_plan_linear(x, wq, sc, bi, group, bits, y)["kernel"] == kernel, (bits, group, N)
            aq.aq_qmm_t(x, wq, sc, bi, group, bits, out=y)
            got = y.double().cpu().numpy()
            assert np.all(np.abs(got - exact) <= 1e-6 * exact), (bits, group, N, got.ravel()[:4], exact)


# ---------------------------------------------------------------------------
# strided batched views (candle pitfall page)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 8])
def test_qk_scores_strided(bits):
    """scores = Q . K^T per (b, h) with K quantized (G = head_dim = 64) as a batched bank."""
    qkv, q, k = inputs.qkv_case()
    Q, (wq, sc, bi) = _q(k.float().contiguous().reshape(-1, 64), 64, bits)
    wq = wq.view(2, 4, 5, -1)
    sc = sc.view(2, 4, 5, 1)
    bi = bi.view(2, 4, 5, 1)
    wd = Q.dequant().reshape(2, 4, 5, 64)
    qkv_d = qkv.to(DEV)
    q_d = qkv_d.narrow(1, 0, 4)
    assert q_d.stride() == (3840, 320, 64, 1)
    y = aq.aq_qmm_t(q_d, wq, sc, bi, 64, bits)
    ref = oracle_linear_view(q, wd)
    err = row_errors(y, ref)
    assert np.all(err <= 4e-3), err
    # the contiguous copy gives the same bits, batch by batch, head by head
    y_c = aq.aq_qmm_t(q_d.contiguous(), wq, sc, bi, 64, bits)
    for b in range(2):
        for h in range(4):
            assert torch.equal(y[b, h], y_c[b, h]), (b, h)


@pytest.mark.parametrize("entry", ["aq_qmm_t", "aq_qmv"])
def test_linear4d_narrowed(entry):
    base, x, w = inputs.linear4d_case()
    Q, (wq, sc, bi) = _q(w, 32, 8)
    wd = Q.dequant()
    base_d = base.to(DEV)
    x_d = base_d.narrow(1, 0, 2)
    fn = getattr(aq, entry)
    y = fn(x_d, wq, sc, bi, 32, 8)
    ref = oracle_linear_view(x, wd)
    assert np.all(row_errors(y, ref) <= 4e-3)
    y_c = fn(x_d.contiguous(), wq, sc, bi, 32, 8)
    for b0 in range(2):
        for b1 in range(2):
            assert torch.equal(y[b0, b1], y_c[b0, b1])


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

def test_empty_rows_launch_nothing():
    w = inputs.normal((64, 256), 1.0, seed=1)
    _, (wq, sc, bi) = _q(w, 64, 4)
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    y = aq.aq_qmm_t(x, wq, sc, bi, 64, 4)
    assert y.shape == (0, 64)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_output_canaries_untouched(bits):
    """Writes stay inside y: guard regions before/after and between strided rows keep their value."""
    N, K, M = 37, 256, 3
    w = inputs.normal((N, K), 1.0, seed=bits + 50)
    Q, (wq, sc, bi) = _q(w, 64, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=51).to(DEV)
    buf = torch.full((M + 2, N + 8), 3072.0, dtype=torch.bfloat16, device=DEV)
    y = buf[1:M + 1, 4:4 + N]
    aq.aq_qmm_t(x, wq, sc, bi, 64, bits, out=y)
    b = buf.float().cpu()
    assert torch.all(b[0] == 3072.0) and torch.all(b[-1] == 3072.0)
    assert torch.all(b[:, :4] == 3072.0) and torch.all(b[:, 4 + N:] == 3072.0)
    ref = oracle_linear_view(x.cpu(), Q.dequant())
    assert np.all(row_errors(y, ref) <= 4e-3)


def _gemv_fp32_bound(Q, x: torch.Tensor, bits: int) -> np.ndarray:
    """Worst-case fp32 error of the GEMV's fp32 output, per element (forward error analysis).

    Per 32-code chunk the GEMV adds 32 exact products (BASE + q) * x (BASE = 128, or 256 for
    8-bit codes) and the 32 widened x values, then folds s * P + (b - BASE*s) * X into the row
    sum; the chunk sums of all lanes meet in a 5-level shuffle tree.  With u = 2^-24 every
    rounded sum of n terms is off by at most n*u times the sum of their magnitudes, so
        |y - ref| <= (32 + C + 8) * u * sum_k (|s_k| (BASE + q_k) + |b_k| + BASE |s_k|) |x_k|
    with C the number of chunks.  This is an absolute bound: the offset BASE makes it scale with
    BASE * |s| * sum|x|, not with |y|.
    """
    base = 256.0 if bits == 8 else 128.0
    G = Q.group
    s = np.repeat(oracle.half_to_double(Q.scale_bits, "bf16"), G, axis=-1)
    b = np.repeat(oracle.half_to_double(Q.bias_bits, "bf16"), G, axis=-1)
    mag = np.abs(s) * (base + Q.codes) + np.abs(b) + base * np.abs(s)          # [N, K]
    xa = np.abs(x.float().double().numpy().reshape(-1, x.shape[-1]))          # [M, K]
    C = x.shape[-1] // 32
    return (32 + C + 8) * 2.0 ** -24 * (xa @ mag.T)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [32, 4096])
def test_gemv_fp32_output_bound(bits, K):
    """fp32 outputs of the GEMV stay inside their derived rounding bound (single row, K from one
    chunk to 128 chunks)."""
    w = inputs.normal((3, K), 1.0, seed=77 + K)
    Q, (wq, sc, bi) = _q(w, 32, bits)
    x = inputs.normal((1, K), 1.0, torch.bfloat16, seed=78 + K)
    y = aq.aq_qmv(x.to(DEV), wq, sc, bi, 32, bits, out_dtype=torch.float32)
    ref = oracle_linear_view(x, Q.dequant())
    bound = _gemv_fp32_bound(Q, x, bits)
    assert np.all(np.abs(y.double().cpu().numpy() - ref) <= bound), (y, ref, bound)


def test_f16_activations():
    w = inputs.normal((300, 1024), 0.02, seed=5)
    Q, (wq, sc, bi) = _q(w, 64, 4, "f16")
    x = inputs.normal((3, 1024), 1.0, torch.float16, seed=6)
    y = aq.aq_qmm_t(x.to(DEV), wq, sc, bi, 64, 4)
    ref = oracle_linear_view(x, Q.dequant())
    assert np.all(row_errors(y, ref) <= 4e-3)
