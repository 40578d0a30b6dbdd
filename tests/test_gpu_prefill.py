"""GPU parity of the prefill tensor-core kernel (rows per launch >= 64, groups 64/128:
tiles of 128 W rows x 128 tokens) against the oracle.

Several token tiles with a ragged tail, ragged W rows, K from one stage to two scale/bias
chunks, every supported bit width, both activation dtypes, fp32 outputs, batched and strided
views, and the prefill shapes of the decoder MLP at full size on sampled rows.
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


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("M,N,K", [(64, 128, 256), (130, 300, 512), (257, 200, 4096)])
def test_prefill_shapes(bits, group, M, N, K):
    w = inputs.normal((N, K), 0.02, seed=M + N + K + bits + group)
    Q, (wq, sc, bi) = _q(w, group, bits)
    x = inputs.normal((M, K), 1.0, torch.bfloat16, seed=M * 3 + K)
    xd = x.to(DEV)
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    err = row_errors(y, oracle_linear_view(x, Q.dequant()))
    assert np.all(err <= 4e-3), (err.max(), int(err.argmax()))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
def test_prefill_dtypes_fp32_out(bits, xdtype):
    M, N, K, group = 200, 260, 2048, 64
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    w = inputs.normal((N, K), 0.02, seed=bits + 7)
    Q, (wq, sc, bi) = _q(w, group, bits, sd)
    x = inputs.normal((M, K), 1.0, xdtype, seed=bits + 8)
    xd = x.to(DEV)
    ref = oracle_linear_view(x, Q.dequant())
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    assert np.all(row_errors(y, ref) <= 4e-3)
    # fp32 output: only fp32 summation order remains
    y32 = aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out_dtype=torch.float32)
    assert np.all(row_errors(y32, ref) <= 1e-4)


def test_prefill_batched_views():
    """Non-foldable batch dims with >= 64 rows each: every batch element matches the contiguous
    copy bit for bit and the oracle to the bar."""
    K, N, bits, group = 1024, 300, 4, 64
    w = inputs.normal((N, K), 0.02, seed=51)
    Q, (wq, sc, bi) = _q(w, group, bits)
    base = inputs.normal((3, 2, 100, K), 1.0, torch.bfloat16, seed=52)
    x = base.narrow(2, 10, 70)                     # [3, 2, 70, K]: rows do not fold across batches
    xd = base.to(DEV).narrow(2, 10, 70)
    y = aq.aq_qmm_t(xd, wq, sc, bi, group, bits)
    yc = aq.aq_qmm_t(xd.contiguous(), wq, sc, bi, group, bits)
    assert torch.equal(y, yc)
    assert np.all(row_errors(y, oracle_linear_view(x, Q.dequant())) <= 4e-3)


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("M,N", [(200, 1000), (128, 128), (70, 300), (70, 1)])
def test_prefill_y_tile_store_stays_inside_y(xdtype, group, M, N):
    """With N a multiple of 8 and 16-byte aligned rows of y each 128 x 128 tile leaves as one bulk
    tensor store of a shared-memory tile (groups of 64; N 300 and 1, and groups of 128, whose W
    ring would get too shallow, take element stores): guard columns and rows around
    a strided y keep their value, ragged tiles write nothing outside y, batch elements of a padded
    batched y stay apart, and the values are bitwise those of the element-wise stores taken when y's
    row stride is not a multiple of 8."""
    K, bits = 1024, 4
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    w = inputs.normal((N, K), 0.02, seed=M + N + group)
    Q, (wq, sc, bi) = _q(w, group, bits, sd)
    x = inputs.normal((M, K), 1.0, xdtype, seed=M * 5 + N)
    xd = x.to(DEV)
    pitch = (N + 15) // 8 * 8 + 8                  # row stride a multiple of 8 elements: tile stores
    buf = torch.full((M + 2, pitch + 8), 3072.0, dtype=xdtype, device=DEV)
    y = buf[1:M + 1, 8:8 + N]
    assert aq.aq_plan_linear(xd, wq, sc, bi, group, bits, y)["kernel"] == "tc_prefill"
    aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out=y)
    b = buf.float().cpu()
    assert torch.all(b[0] == 3072.0) and torch.all(b[-1] == 3072.0)
    assert torch.all(b[:, :8] == 3072.0) and torch.all(b[:, 8 + N:] == 3072.0)
    assert np.all(row_errors(y, oracle_linear_view(x, Q.dequant())) <= 4e-3)
    odd = torch.full((M, N + 1), 3072.0, dtype=xdtype, device=DEV)[:, :N]   # stride N + 1: element stores
    aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out=odd)
    assert torch.equal(odd, y)
    xb = inputs.normal((2, M, K), 1.0, xdtype, seed=M + 9).to(DEV)
    ybuf = torch.full((2, M + 3, pitch), 3072.0, dtype=xdtype, device=DEV)
    yb = ybuf[:, :M, :N]
    aq.aq_qmm_t(xb, wq, sc, bi, group, bits, out=yb)
    assert torch.all(ybuf[:, M:].float() == 3072.0) and torch.all(ybuf[:, :, N:].float() == 3072.0)
    for i in range(2):
        assert torch.equal(yb[i], aq.aq_qmm_t(xb[i].contiguous(), wq, sc, bi, group, bits))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("shape", ["up", "down"])
def test_prefill_full_size_every_batch_element(bits, shape):
    """x [8, 2048, K] against the decoder MLP's W [14336, 4096] (up) or [4096, 14336] (down) at
    full size, in the one launch the benchmark times.

    Every row is checked: the whole y (bf16, tcgen05 prefill kernel) against the same call through
    the CUDA-core GEMV with fp32 output (independent code, no tensor cores), by the per-row bar.
    Both are anchored to the fp64 oracle on the first and last token and two seeded tokens of
    every 128-token tile of every batch element (34 rows per batch element), every column.
    """
    if shape == "up":
        xs, (N, K) = inputs.PREFILL_X, inputs.PREFILL_W_UP
    else:
        xs, (N, K) = inputs.PREFILL_X_DOWN, inputs.PREFILL_W_DOWN
    group = inputs.PREFILL_GROUP
    B, S = xs[0], xs[1]
    w = inputs.normal((N, K), 0.02, seed=61 + bits)
    Q, (wq, sc, bi) = _q(w, group, bits)
    del w
    xd = inputs.normal(xs, 1.0, torch.bfloat16, seed=62, device=DEV)
    y = torch.empty(xs[:-1] + (N,), dtype=torch.bfloat16, device=DEV)
    assert aq.aq_plan_linear(xd, wq, sc, bi, group, bits, y)["kernel"] == "tc_prefill"
    aq.aq_qmm_t(xd, wq, sc, bi, group, bits, out=y)
    y_ind = aq.aq_qmv(xd, wq, sc, bi, group, bits, out_dtype=torch.float32)
    torch.cuda.synchronize()
    # every row of every batch element against the independent kernel
    for b in range(B):
        err = row_errors(y[b], y_ind[b].double().cpu().numpy())
        assert err.size == S and np.all(err <= 4e-3), (b, err.max(), int(err.argmax()))
    # the oracle on sampled rows of every tile of every batch element
    g = np.random.default_rng(bits * 10 + len(shape))
    rows = []
    for b in range(B):
        rows += [(b, 0), (b, S - 1)]
        for t0 in range(0, S, 128):
            rows += [(b, t0 + int(r)) for r in g.choice(128, size=2, replace=False)]
    wd = Q.dequant()
    xb = torch.stack([xd[b, t] for b, t in rows]).cpu()
    ref = oracle.linear_contig(xb.view(torch.int16).numpy().view(np.uint16), "bf16", wd)
    got = torch.stack([y[b, t] for b, t in rows])
    got_ind = torch.stack([y_ind[b, t] for b, t in rows])
    assert np.all(row_errors(got, ref) <= 4e-3)
    assert np.all(row_errors(got_ind, ref) <= 4e-3)
