"""GPU parity of the gathered GEMV (aq_qmv_gathered: per-row token and expert ids read on the
device, no host-side sort) against the oracle.

Expert banks of the "Metal Kernel Bits=8 Final Report" expert shapes (section 4.3: [2816 out,
1408 in], 8-bit, G = 32) on a reduced number of experts, and a 4-bit G = 64 bank with f16
activations; tokens routed to distinct experts uniformly at random (top-k).  Every row is
checked against x[token] . dequant(W[expert])^T in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_qmv_b200 import aq, inputs
from tests.parity import dtype_name, half_bits, row_errors, to_device_quant

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _bank(E, N, K, group, bits, sdtype, seed):
    Q = oracle.quantize(inputs.normal((E, N, K), 0.02, seed=seed).numpy(), group, bits, sdtype)
    tdt = torch.bfloat16 if sdtype == "bf16" else torch.float16
    return Q, to_device_quant(Q, DEV, tdt)


def _expected(Q, x, x_ids, w_ids):
    xb = half_bits(x)
    wd = Q.dequant()
    return np.stack([oracle.linear_contig(xb[t:t + 1], dtype_name(x), wd[e])[0]
                     for t, e in zip(x_ids.tolist(), w_ids.tolist())])


@pytest.mark.parametrize("bits,group,xdtype,E,N,K", [(8, 32, torch.bfloat16, 16, 2816, 1408),
                                                      (4, 64, torch.float16, 12, 1000, 1024),
                                                      (2, 128, torch.bfloat16, 8, 257, 512),
                                                      (3, 32, torch.bfloat16, 8, 130, 256)])
def test_gathered_rows_match_oracle(bits, group, xdtype, E, N, K):
    T, topk = 5, 4
    routing = inputs.moe_routing(tokens=T, experts=E, topk=topk, seed=bits)
    x_ids = torch.arange(T).repeat_interleave(topk)
    w_ids = routing.reshape(-1)
    Q, (wq, sc, bi) = _bank(E, N, K, group, bits, dtype_name(torch.empty(0, dtype=xdtype)), seed=bits + 40)
    x = inputs.normal((T, K), 1.0, xdtype, seed=bits + 41)
    y = aq.aq_qmv_gathered(x.to(DEV), x_ids.to(DEV), w_ids.to(DEV), wq, sc, bi, group, bits)
    aq.aq_device_error()
    ref = _expected(Q, x, x_ids, w_ids)
    err = row_errors(y, ref)
    assert err.size == T * topk and np.all(err <= 4e-3), (err.max(), int(err.argmax()))
    # fp32 output against the same rows
    y32 = aq.aq_qmv_gathered(x.to(DEV), x_ids.to(DEV), w_ids.to(DEV), wq, sc, bi, group, bits,
                             out_dtype=torch.float32)
    assert np.all(row_errors(y32, ref) <= 1e-4)


def test_gathered_bad_ids_flagged():
    E, N, K, group, bits = 4, 64, 256, 64, 4
    Q, (wq, sc, bi) = _bank(E, N, K, group, bits, "bf16", seed=3)
    x = inputs.normal((3, K), 1.0, torch.bfloat16, seed=4)
    x_ids = torch.tensor([0, 3, 1, 2, -1])
    w_ids = torch.tensor([1, 0, 4, 3, 2])
    y = aq.aq_qmv_gathered(x.to(DEV), x_ids.to(DEV), w_ids.to(DEV), wq, sc, bi, group, bits)
    with pytest.raises(aq.AQError) as ei:
        aq.aq_device_error()
    assert ei.value.name == "AQ_ERR_INDEX"
    got = y.float().cpu()
    for bad in (1, 2, 4):
        assert torch.all(got[bad] == 0), bad
    good = [0, 3]
    ref = _expected(Q, x, x_ids[good], w_ids[good])
    assert np.all(row_errors(y[good], ref) <= 4e-3)
    aq.aq_device_error()   # cleared by the read above


def test_gathered_matches_grouped_kernel_rows():
    """The same routed rows through the sorted-bank tensor-core entry point and through the
    gathered GEMV: both within the bar of the oracle, row for row (different kernels)."""
    E, N, K, group, bits = 16, inputs.MOE_N, inputs.MOE_K, inputs.MOE_GROUP, inputs.MOE_BITS
    T, topk = 12, 4
    routing = inputs.moe_routing(tokens=T, experts=E, topk=topk, seed=8)
    tok, offsets = inputs.moe_sort(routing, E)
    Q, (wq, sc, bi) = _bank(E, N, K, group, bits, "bf16", seed=9)
    x = inputs.normal((T, K), 1.0, torch.bfloat16, seed=10)
    exp_of_row = torch.repeat_interleave(torch.arange(E), offsets[1:] - offsets[:-1])
    y_g = aq.aq_qmv_gathered(x.to(DEV), tok.to(DEV), exp_of_row.to(DEV), wq, sc, bi, group, bits)
    y_s = aq.aq_qmm_t_grouped(x[tok].contiguous().to(DEV), offsets.to(DEV), wq, sc, bi, group, bits)
    ref = _expected(Q, x, tok, exp_of_row)
    assert np.all(row_errors(y_g, ref) <= 4e-3)
    assert np.all(row_errors(y_s, ref) <= 4e-3)
