"""GPU parity of the tcgen05 tensor-core regime (rows per launch > 4) against the oracle.

Covers several tiles and ragged tails in every dimension: tokens (M not a
multiple of 16), W rows (N not a multiple of 128), K from one stage (64) to
many, every supported bit width, group size and activation dtype, strided and
batched x views, fp32 outputs, and the grouped (mixture-of-experts) entry point
with empty and uneven experts.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_qmv_b200 import aq, inputs
from tests.parity import dtype_name, oracle_linear_view, row_errors, to_device_quant

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _q(w, group, bits, sdtype="bf16"):
    Q = oracle.quantize(w.float().numpy(), group, bits, sdtype)
    tdt = torch.bfloat16 if sdtype == "bf16" else torch.float16
    return Q, to_device_quant(Q, DEV, tdt)


def _regime(x, wq, sc, bi, group, bits):
    y = torch.empty(tuple(x.shape[:-1]) + (wq.shape[-2],), dtype=x.dtype, device=x.device)
    return aq.aq_plan_linear(x, wq, sc, bi, group, bits, y)["regime"]


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
@pytest.mark.parametrize("M,N,K", [(5, 129, 128), (16, 128, 128), (17, 300, 256), (32, 1000, 1024),
                                   (33, 257, 512), (64, 640, 1024), (100, 200, 256), (256, 384, 640),
                                   (300, 131, 384)])
def test_mma_shapes(bits, M, N, K):
    group = 64
    w = inputs.normal((N, K), 0.02, seed=M * 7 + N + K + bits)
    Q, (wq, sc, bi) = _q(w, group, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=M + K)
    xd = x.to(DEV)
    assert _regime(xd, wq, sc, bi, group, bits) == "mma"
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    ref = oracle_linear_view(x, Q.dequant())
    err = row_errors(y, ref)
    assert np.all(err <= 4e-3), (err.max(), int(err.argmax()))


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [4, 8])
def test_mma_groups_dtypes(group, xdtype, bits):
    M, N, K = 24, 260, 4096   # K spans several scale/bias chunks for every group size
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    w = inputs.normal((N, K), 0.02, seed=group + bits)
    Q, (wq, sc, bi) = _q(w, group, bits, sd)
    x = inputs.normal((M, K), 1.0, xdtype, seed=group * 3 + bits)
    xd = x.to(DEV)
    assert _regime(xd, wq, sc, bi, group, bits) == "mma"
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    ref = oracle_linear_view(x, Q.dequant())
    assert np.all(row_errors(y, ref) <= 4e-3)
    # fp32 output: no weight rounding anywhere, only fp32 summation order remains
    y32 = aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out_dtype=torch.float32)
    assert np.all(row_errors(y32, ref) <= 1e-4)


def test_mma_batched_and_strided_views():
    """Non-foldable batch dims (launch batches), a row-strided x and a strided y."""
    K, N, bits, group = 512, 200, 4, 64
    w = inputs.normal((N, K), 0.02, seed=5)
    Q, (wq, sc, bi) = _q(w, group, bits)
    wd = Q.dequant()
    base = inputs.normal((3, 4, 9, K), 1.0, torch.bfloat16, seed=6)
    x = base.narrow(1, 1, 2)                      # [3, 2, 9, K], batch dim 0 does not fold
    xd = base.to(DEV).narrow(1, 1, 2)
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    ref = oracle_linear_view(x, wd)
    assert np.all(row_errors(y, ref) <= 4e-3)
    # same bits as the contiguous copy, every batch element
    yc = aq.aq_qmm_t(xd.contiguous(), wq, sc, bi, group, bits)
    for b0 in range(3):
        for b1 in range(2):
            assert torch.equal(y[b0, b1], yc[b0, b1])
    # every other row of a 2D x, written into every other row of a wider y
    base2 = inputs.normal((40, K), 1.0, torch.bfloat16, seed=7)
    x2 = base2[::2]
    ybuf = torch.zeros(20, 2 * N, dtype=torch.bfloat16, device=DEV)
    y2 = ybuf[:, :N]
    aq.aq_qmm_t(base2.to(DEV)[::2], wq, sc, bi, group, bits, out=y2)
    assert torch.all(ybuf[:, N:] == 0)
    assert np.all(row_errors(y2, oracle_linear_view(x2, wd)) <= 4e-3)


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N", [(37, 5000), (40, 5001), (48, 9728)])
def test_mma_y_tile_store_stays_inside_y(xdtype, M, N):
    """Tiles of y leave through shared memory and one bulk tensor store each when N is a multiple of
    8 and y's rows and batch strides are 16-byte aligned (N 5000: a ragged last W tile; N 5001: the
    element stores instead).  Guard columns and rows around a strided y keep their value, tokens past
    M are not written, padded batch elements stay apart, and the values are bitwise those of the
    element-wise stores taken when y's row stride is not a multiple of 8 elements.  (Enough W tiles
    that K is not split over clusters, which stores y its own way.)"""
    K, bits, group = 1024, 4, 64
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    w = inputs.normal((N, K), 0.02, seed=M + N)
    Q, (wq, sc, bi) = _q(w, group, bits, sd)
    x = inputs.normal((M, K), 1.0, xdtype, seed=M * 3 + N)
    xd = x.to(DEV)
    pitch = (N + 15) // 8 * 8 + 8                  # row stride a multiple of 8 elements
    buf = torch.full((M + 2, pitch + 8), 3072.0, dtype=xdtype, device=DEV)
    y = buf[1:M + 1, 8:8 + N]
    assert aq.aq_plan_linear(xd, wq, sc, bi, group, bits, y)["kernel"] == "tc_small_m"
    aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out=y)
    b = buf.float().cpu()
    assert torch.all(b[0] == 3072.0) and torch.all(b[-1] == 3072.0)
    assert torch.all(b[:, :8] == 3072.0) and torch.all(b[:, 8 + N:] == 3072.0)
    rows = np.r_[0:4, N - 132:N]                   # the first rows and the ragged last W tile
    ysel = y.index_select(1, torch.as_tensor(rows, device=DEV))
    assert np.all(row_errors(ysel, oracle_linear_view(x, Q.dequant()[rows])) <= 4e-3)
    odd = torch.full((M, N + 1), 3072.0, dtype=xdtype, device=DEV)[:, :N]   # stride N + 1: element stores
    aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out=odd)
    assert torch.equal(odd, y)
    xb = inputs.normal((2, M, K), 1.0, xdtype, seed=M + 5).to(DEV)
    ybuf = torch.full((2, M + 3, pitch), 3072.0, dtype=xdtype, device=DEV)
    yb = ybuf[:, :M, :N]
    aq.aq_qmm_t(xb, wq, sc, bi, group, bits, out=yb)
    assert torch.all(ybuf[:, M:].float() == 3072.0) and torch.all(ybuf[:, :, N:].float() == 3072.0)
    for i in range(2):
        assert torch.equal(yb[i], aq.aq_qmm_t(xb[i].contiguous(), wq, sc, bi, group, bits))


def _plan(x, wq, sc, bi, group, bits, y=None):
    if y is None:
        y = torch.empty(tuple(x.shape[:-1]) + (wq.shape[-2],), dtype=x.dtype)
    return aq.aq_plan_linear(x, wq, sc, bi, group, bits, y)


def _empty_weights(N, K, bits, group, dtype=torch.bfloat16):
    """Uninitialised weight views: the plan reads shapes, strides and pointers only."""
    return (torch.empty(N, K * bits // 32, dtype=torch.int32), torch.empty(N, K // group, dtype=dtype),
            torch.empty(N, K // group, dtype=dtype))


def test_plan_reports_tile_stores_of_y():
    """Where the tcgen05 kernels write each tile of y with one bulk tensor store: y in x's 16-bit
    dtype, N a multiple of 8, 16-byte aligned rows and batch strides, no split of K over a cluster,
    and (prefill) room in shared memory; elsewhere element stores.  The warp-level kernel and the
    GEMV never do.  (A host-side plan on CPU tensors; the tensor-core kernels are planned only
    where the driver offers cuTensorMapEncodeTiled, hence a GPU test.)"""
    K = 1024
    lm = _empty_weights(151936, K, 4, 64)
    x32 = torch.zeros(32, 1, K, dtype=torch.bfloat16)
    p = _plan(x32, *lm, 64, 4)
    assert p["kernel"] == "tc_small_m" and p["y_tiles"], p
    p = _plan(x32, *lm, 64, 4, y=torch.empty(32, 1, 151936, dtype=torch.float32))
    assert p["kernel"] == "tc_small_m" and not p["y_tiles"]        # fp32 y
    odd = _empty_weights(151932 + 1, K, 4, 64)
    assert not _plan(x32, *odd, 64, 4)["y_tiles"]                      # N not a multiple of 8
    ypad = torch.empty(32, 151936 + 4, dtype=torch.bfloat16)[:, :151936].unsqueeze(1)
    assert not _plan(x32, *lm, 64, 4, y=ypad)["y_tiles"]               # row stride not a multiple of 8
    small = _empty_weights(304, K, 4, 64)
    p = _plan(torch.zeros(40, K, dtype=torch.bfloat16), *small, 64, 4)
    assert p["kernel"] == "tc_small_m" and not p["y_tiles"]          # few tiles: K split over a cluster
    up = _empty_weights(4096, K, 4, 64)
    xp = torch.zeros(2, 128, K, dtype=torch.bfloat16)
    p = _plan(xp, *up, 64, 4)
    assert p["kernel"] == "tc_prefill" and p["y_tiles"], p
    p = _plan(xp.half(), *_empty_weights(4096, K, 8, 64, torch.float16), 64, 8)
    assert p["kernel"] == "tc_prefill" and p["y_tiles"], p
    # groups of 128: the 32 KB staging tile would leave the W ring too shallow
    p = _plan(xp, *_empty_weights(4096, K, 4, 128), 128, 4)
    assert p["kernel"] == "tc_prefill" and not p["y_tiles"], p
    assert not _plan(xp, *_empty_weights(4100, K, 4, 64), 64, 4)["y_tiles"]
    assert _plan(torch.zeros(8, K, dtype=torch.bfloat16), *up, 64, 4)["kernel"] == "warp_mma"
    assert not _plan(torch.zeros(8, K, dtype=torch.bfloat16), *up, 64, 4)["y_tiles"]
    assert not _plan(torch.zeros(2, K, dtype=torch.bfloat16), *up, 64, 4)["y_tiles"]   # GEMV


@pytest.mark.parametrize("bits", [4, 8])
def test_mma_matches_gemv_numerics(bits):
    """The two regimes agree with each other to the same bar (different kernels)."""
    M, N, K, group = 8, 512, 1024, 64
    w = inputs.normal((N, K), 0.02, seed=11)
    _, (wq, sc, bi) = _q(w, group, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=12).to(DEV)
    a = aq.aq_qmm_t(x, wq, sc, bi, group, bits, out_dtype=torch.float32)
    b = aq.aq_qmv(x, wq, sc, bi, group, bits, out_dtype=torch.float32)
    rel = ((a - b).abs().amax(-1) / b.abs().amax(-1)).max().item()
    assert rel <= 4e-3


@pytest.mark.parametrize("bits", [4, 8])
def test_grouped_experts(bits):
    E, N, K, group = 6, 200, 256, 32
    counts = [5, 0, 17, 1, 40, 9]
    T = sum(counts)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    w = inputs.normal((E, N, K), 0.02, seed=21)
    Q = oracle.quantize(w.numpy(), group, bits, "bf16")
    wq, sc, bi = to_device_quant(Q, DEV, torch.bfloat16)
    x = inputs.normal((T, K), 1.0, torch.bfloat16, seed=22)
    off_d = torch.from_numpy(offsets).to(DEV)
    y = aq.aq_qmm_t_grouped(x.to(DEV), off_d, wq, sc, bi, group, bits)
    xb = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.linear_grouped(xb, "bf16", offsets, Q.dequant())
    assert np.all(row_errors(y, ref) <= 4e-3)


def test_grouped_moe_bank_shape():
    """Expert bank of the "Metal Kernel Bits=8 Final Report" shapes (8-bit, G=32,
    [2816 out, 1408 in]) on a reduced number of experts, routed top-8 at random."""
    E, N, K, group, bits = 16, inputs.MOE_N, inputs.MOE_K, inputs.MOE_GROUP, inputs.MOE_BITS
    routing = inputs.moe_routing(tokens=24, experts=E, topk=4, seed=3)
    tok, offsets = inputs.moe_sort(routing, E)
    w = inputs.normal((E, N, K), 0.02, seed=31)
    Q = oracle.quantize(w.numpy(), group, bits, "bf16")
    wq, sc, bi = to_device_quant(Q, DEV, torch.bfloat16)
    x_tok = inputs.normal((24, K), 1.0, torch.bfloat16, seed=32)
    x_sorted = x_tok[tok].contiguous()
    y = aq.aq_qmm_t_grouped(x_sorted.to(DEV), offsets.to(DEV), wq, sc, bi, group, bits)
    # oracle on a sample of 3 rows per expert segment, all columns
    wd = Q.dequant()
    xb = x_sorted.view(torch.int16).numpy().view(np.uint16)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        for r in list(range(lo, min(hi, lo + 3))):
            ref = oracle.linear_contig(xb[r:r + 1], "bf16", wd[e])
            assert np.all(row_errors(y[r:r + 1], ref) <= 4e-3), (e, r)


def test_grouped_moe_bank_config_size():
    """The full expert bank of the benchmark: 128 experts of [2816 out, 1408 in], 8-bit, G = 32
    ("Metal Kernel Bits=8 Final Report" shapes), 256 tokens routed to 8 distinct experts each
    (2048 rows), one launch; every row against every column of the fp64 oracle."""
    E, N, K, group, bits = inputs.MOE_EXPERTS, inputs.MOE_N, inputs.MOE_K, inputs.MOE_GROUP, inputs.MOE_BITS
    tok, offsets = inputs.moe_sort(inputs.moe_routing())
    T = tok.numel()
    x_tok = inputs.normal((inputs.MOE_TOKENS, K), 1.0, torch.bfloat16, seed=9)
    x_sorted = x_tok[tok].contiguous()
    xb = x_sorted.view(torch.int16).numpy().view(np.uint16)
    wq = torch.empty(E, N, K * bits // 32, dtype=torch.int32, device=DEV)
    sc = torch.empty(E, N, K // group, dtype=torch.bfloat16, device=DEV)
    bi = torch.empty_like(sc)
    ref = np.empty((T, N), np.float64)
    for e in range(E):
        Q = oracle.quantize(inputs.normal((N, K), inputs.W_STD, seed=100 + e).numpy(), group, bits, "bf16")
        qd = to_device_quant(Q, DEV, torch.bfloat16)
        wq[e].copy_(qd[0]); sc[e].copy_(qd[1]); bi[e].copy_(qd[2])
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            ref[lo:hi] = oracle.linear_contig(xb[lo:hi], "bf16", Q.dequant())
    y = aq.aq_qmm_t_grouped(x_sorted.to(DEV), offsets.to(DEV), wq, sc, bi, group, bits)
    err = row_errors(y, ref)
    assert err.size == T == 2048 and np.all(err <= 4e-3), (err.max(), int(err.argmax()))


def test_grouped_offsets_clamped_on_device():
    """Offsets the host cannot check (they live on the device) that start below 0 and end past T:
    the kernel clamps each expert's rows into [0, T), writes nothing outside y_sorted (canary rows
    and columns around it keep their value) and the rows it owns match the oracle."""
    E, N, K, group, bits = 4, 200, 256, 32, 8
    T = 40
    bad = np.array([-7, 10, 25, 25, 60], np.int64)
    clamped = np.array([0, 10, 25, 25, 40], np.int64)
    w = inputs.normal((E, N, K), 0.02, seed=71)
    Q = oracle.quantize(w.numpy(), group, bits, "bf16")
    wq, sc, bi = to_device_quant(Q, DEV, torch.bfloat16)
    x = inputs.normal((T, K), 1.0, torch.bfloat16, seed=72)
    buf = torch.full((T + 4, N + 8), 3072.0, dtype=torch.bfloat16, device=DEV)
    y = buf[2:T + 2, 4:4 + N]
    aq.aq_qmm_t_grouped(x.to(DEV), torch.from_numpy(bad).to(DEV), wq, sc, bi, group, bits, out=y)
    aq.aq_device_error()
    b = buf.float().cpu()
    assert torch.all(b[:2] == 3072.0) and torch.all(b[T + 2:] == 3072.0)
    assert torch.all(b[:, :4] == 3072.0) and torch.all(b[:, 4 + N:] == 3072.0)
    xb = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.linear_grouped(xb, "bf16", clamped, Q.dequant())
    assert np.all(row_errors(y, ref) <= 4e-3)


def test_odd_group_count_takes_gemv():
    """K/group odd (K=192, G=64) is served by the GEMV kernel, still to the same bar."""
    w = inputs.normal((100, 192), 0.02, seed=41)
    Q, (wq, sc, bi) = _q(w, 64, 4)
    x = inputs.normal((20, 192), 1.0, torch.bfloat16, seed=42)
    xd = x.to(DEV)
    assert _regime(xd, wq, sc, bi, 64, 4) == "qmv"
    y = aq.aq_qmm_t(xd, wq, sc, bi, 64, 4)
    assert np.all(row_errors(y, oracle_linear_view(x, Q.dequant())) <= 4e-3)


def test_device_error_word_clear():
    aq.aq_device_error()


def test_bounded_wait_reports_timeout():
    """A bounded wait that runs out (on a barrier nothing completes, 2 ms budget) is reported as
    AQ_ERR_TIMEOUT by aq_device_error, which clears it; the device stays usable and the next
    call is correct with a clean error word."""
    aq.aq_device_error()
    aq.aq_check_bounded_wait(2_000_000)
    with pytest.raises(aq.AQError) as ei:
        aq.aq_device_error()
    assert ei.value.name == "AQ_ERR_TIMEOUT"
    assert "bounded-wait self-check" in str(ei.value)   # the wait that expired is named
    aq.aq_device_error()
    M, N, K, group, bits = 40, 300, 512, 64, 4
    w = inputs.normal((N, K), 0.02, seed=81)
    Q, (wq, sc, bi) = _q(w, group, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=82)
    y = aq.aq_qmm_t(x.to(DEV), wq, sc, bi, group, bits)
    aq.aq_device_error()
    assert np.all(row_errors(y, oracle_linear_view(x, Q.dequant())) <= 4e-3)
