"""GPU parity of the warp-level mma.sync kernel (5..32 rows of x in total, 2/4/8-bit codes)
against the oracle.

Ragged tokens (every n8 tile count, M not a multiple of 8), ragged W rows (N = 1, odd N, N not
a multiple of 32), K from one group pair to 4096, every group size and both activation dtypes,
fp32 outputs, batched and strided views (bit for bit equal to the contiguous copy), strided y,
the kernel choice between the warp and the tcgen05 kernels, and every matrix of the decode
step at full size, lm_head included, on all rows.
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


def _kernel(x, wq, sc, bi, group, bits):
    y = torch.empty(tuple(x.shape[:-1]) + (wq.shape[-2],), dtype=x.dtype, device=x.device)
    return aq.aq_plan_linear(x, wq, sc, bi, group, bits, y)["kernel"]


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(5, 129, 128), (8, 40, 256), (9, 1, 256), (13, 300, 384), (16, 1000, 1024),
                                   (17, 33, 512), (24, 4099, 1024), (32, 300, 1024), (16, 257, 3072),
                                   (8, 5000, 4096), (13, 300, 640), (32, 1000, 3072),
                                   (16, 4096, 8192)])   # x tile too large for shared memory: read through L1
def test_warp_shapes(bits, M, N, K):
    group = 64
    w = inputs.normal((N, K), 0.02, seed=M * 5 + N + K + bits)
    Q, (wq, sc, bi) = _q(w, group, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=M + 3 * K)
    xd = x.to(DEV)
    assert _kernel(xd, wq, sc, bi, group, bits) == "warp_mma"
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    err = row_errors(y, oracle_linear_view(x, Q.dequant()))
    assert np.all(err <= 4e-3), (err.max(), int(err.argmax()))


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_warp_groups_dtypes(group, xdtype, bits):
    M, N, K = 16, 260, 4096
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    w = inputs.normal((N, K), 0.02, seed=group + bits + 100)
    Q, (wq, sc, bi) = _q(w, group, bits, sd)
    x = inputs.normal((M, K), 1.0, xdtype, seed=group * 3 + bits + 100)
    xd = x.to(DEV)
    # 2-bit codes in groups of 32 leave a lane half a word: the tcgen05 kernel takes them
    expect = "tc_small_m" if (bits == 2 and group == 32) else "warp_mma"
    assert _kernel(xd, wq, sc, bi, group, bits) == expect
    ref = oracle_linear_view(x, Q.dequant())
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    assert np.all(row_errors(y, ref) <= 4e-3)
    y32 = aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out_dtype=torch.float32)
    assert np.all(row_errors(y32, ref) <= 1e-4)


def test_warp_batched_and_strided_views():
    """Launch batches that do not fold (20 rows in total), their contiguous copy (bit for bit),
    and a strided y."""
    K, N, bits, group = 512, 200, 4, 64
    w = inputs.normal((N, K), 0.02, seed=105)
    Q, (wq, sc, bi) = _q(w, group, bits)
    wd = Q.dequant()
    base = inputs.normal((2, 4, 5, K), 1.0, torch.bfloat16, seed=106)
    x = base.narrow(1, 1, 2)                      # [2, 2, 5, K]
    xd = base.to(DEV).narrow(1, 1, 2)
    assert _kernel(xd, wq, sc, bi, group, bits) == "warp_mma"
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    assert np.all(row_errors(y, oracle_linear_view(x, wd)) <= 4e-3)
    yc = aq.aq_qmm_t(xd.contiguous(), wq, sc, bi, group, bits)
    assert torch.equal(y, yc)
    # every other row of x, into every other column block of a wider y
    base2 = inputs.normal((40, K), 1.0, torch.bfloat16, seed=107)
    ybuf = torch.zeros(20, 2 * N + 1, dtype=torch.bfloat16, device=DEV)
    y2 = ybuf[:, 1:N + 1]                          # odd row stride and odd offset: scalar stores
    aq.aq_qmm_t(base2.to(DEV)[::2], wq, sc, bi, group, bits, out=y2)
    assert torch.all(ybuf[:, 0] == 0) and torch.all(ybuf[:, N + 1:] == 0)
    assert np.all(row_errors(y2, oracle_linear_view(base2[::2], wd)) <= 4e-3)


def test_warp_matches_other_kernels():
    """The warp kernel, the GEMV and the tcgen05 kernel agree to the bar on one problem."""
    M, N, K, group, bits = 32, 512, 1024, 64, 4
    w = inputs.normal((N, K), 0.02, seed=111)
    _, (wq, sc, bi) = _q(w, group, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=112).to(DEV)
    a = aq.aq_qmm_t(x, wq, sc, bi, group, bits, out_dtype=torch.float32)
    b = aq.aq_qmv(x, wq, sc, bi, group, bits, out_dtype=torch.float32)
    c = aq.aq_qmm_t(torch.cat([x, x]), wq, sc, bi, group, bits, out_dtype=torch.float32)[:M]  # 64 rows
    for ref in (b, c):
        rel = ((a - ref).abs().amax(-1) / ref.abs().amax(-1)).max().item()
        assert rel <= 4e-3


def test_warp_kernel_choice():
    """Up to 8 rows always take the warp kernel; 16 rows unless CTAs of eight row blocks would give
    a warp more than eight 64-code sub-blocks of K (lm_head); 32 rows while each warp of a one-row-block CTA has at most four
    once a cluster splits K (every decode projection), the tcgen05 kernel otherwise (lm_head: many
    row blocks per CTA; large K with many row blocks)."""
    def kern(M, K, N):
        x = torch.empty((M, 1, K), dtype=torch.bfloat16, device=DEV)
        wq = torch.empty((N, K // 8), dtype=torch.int32, device=DEV)
        s = torch.empty((N, K // 64), dtype=torch.bfloat16, device=DEV)
        return _kernel(x, wq, s, s, 64, 4)
    assert kern(32, 1024, 2048) == "warp_mma"
    assert kern(32, 1024, 3072) == "warp_mma"
    assert kern(32, 3072, 1024) == "warp_mma"
    assert kern(32, 2048, 1024) == "warp_mma"
    assert kern(32, 8192, 4096) == "tc_small_m"
    assert kern(32, 1024, 151936) == "tc_small_m"
    assert kern(16, 3072, 1024) == "warp_mma"
    assert kern(8, 1024, 151936) == "warp_mma"
    assert kern(16, 1024, 151936) == "tc_small_m"
    assert kern(16, 1024, 4096) == "warp_mma"
    assert kern(4, 1024, 1024) == "gemv"


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("shape", [inputs.DECODE_PROJ[0], inputs.DECODE_PROJ[1], inputs.DECODE_PROJ[4],
                                   inputs.DECODE_PROJ[6], inputs.DECODE_PROJ_ALT_O, inputs.LM_HEAD])
@pytest.mark.parametrize("batch", [32, 8])
def test_decode_full_size(bits, shape, batch):
    """x [batch, 1, K] against every matrix shape of the decode step (whichever kernel the choice
    gives), all rows and columns."""
    name, K, N = shape
    w = inputs.decode_w(K, N, seed=120 + bits)
    Q, (wq, sc, bi) = _q(w, inputs.DECODE_GROUP, bits)
    del w
    x = inputs.decode_x(K, batch=batch, seed=121)
    xd = x.to(DEV)
    assert _kernel(xd, wq, sc, bi, inputs.DECODE_GROUP, bits) in ("warp_mma", "tc_small_m")
    y = aq.aq_qmm_t(xd, wq, sc, bi, inputs.DECODE_GROUP, bits)
    ref = oracle.linear_contig(x.reshape(-1, K).view(torch.int16).numpy().view(np.uint16), "bf16", Q.dequant())
    err = row_errors(y, ref)
    assert np.all(err <= 4e-3), (name, batch, err.max())


@pytest.mark.parametrize("rows", [8, 32, 40, 128])
def test_weights_rewritten_right_before_the_call(rows):
    """The matrix kernels stage their weights before their wait on the previous kernel in the
    stream, and aq_quantize is documented as safe to run right before them: quantize new weights
    into the same buffers and call the matrix op next, eight times on one stream with no
    synchronisation, and compare every result bit for bit with the same call on freshly quantized
    weights after a full synchronisation (8/32 rows: warp kernel, 40: tcgen05 small-M, 128: prefill)."""
    K, N, group, bits = 1024, 2048, 64, 4
    ws = [inputs.decode_w(K, N, seed=300 + i, device=DEV) for i in range(8)]
    x = inputs.normal((rows, K), 1.0, torch.bfloat16, seed=301, device=DEV)
    wq, sc, bi = aq.aq_quantize(ws[0], group, bits)
    expect = {8: "warp_mma", 32: "warp_mma", 40: "tc_small_m", 128: "tc_prefill"}[rows]
    assert _kernel(x, wq, sc, bi, group, bits) == expect
    outs = []
    for w in ws:
        aq.aq_quantize(w, group, bits, out=(wq, sc, bi))
        outs.append(aq.aq_qmm_t(x, wq, sc, bi, group, bits))
    torch.cuda.synchronize()
    for w, y in zip(ws, outs):
        fresh = aq.aq_quantize(w, group, bits)
        torch.cuda.synchronize()
        assert torch.equal(y, aq.aq_qmm_t(x, *fresh, group, bits))
