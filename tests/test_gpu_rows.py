"""GPU parity of the quantized row gather (embedding lookup, aq_dequantize_rows) against the oracle.

The table has the shape of the "Metal Kernel Bits=8 Final Report" embedding (section 4.1:
[262144, 352] uint32 words, [262144, 44] scales): K = 1408, G = 32 at 8 bits and K = 2816,
G = 64 at 4 bits.  Its codes are random words and its scales and biases random half values
(drawn by the seeded generator, not by either quantizer), so both sides start from the same
table.  Every gathered element must equal the oracle's fp64 dequantization rounded as the
kernel rounds (to fp32, then to the output dtype): bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_qmv_b200 import aq, inputs
from tests.parity import half_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _expected(wq, sc, bi, K, group, bits, ids, sd, out_dtype):
    rows = wq[ids].numpy().view(np.uint32)
    codes = oracle.unpack(rows, K, bits)
    ref = oracle.dequant(codes, half_bits(sc[ids]), half_bits(bi[ids]), group, sd)
    ref32 = ref.astype(np.float32)   # the kernel's one fp32 rounding of s*q + b
    if out_dtype == torch.float32:
        return ref32.view(np.uint32)
    return oracle.float_to_half_bits(ref32, {torch.bfloat16: "bf16", torch.float16: "f16"}[out_dtype])


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32, torch.float16])
def test_embedding_rows_bit_exact(bits, out_dtype):
    sdt = torch.float16 if out_dtype == torch.float16 else torch.bfloat16
    sd = "f16" if sdt == torch.float16 else "bf16"
    wq, sc, bi, K, group = inputs.embedding_table(bits, sdtype=sdt, seed=bits)
    g = inputs.gen(17 + bits)
    ids = torch.cat([torch.tensor([0, inputs.EMBED_ROWS - 1, 12345, 12345]),
                     torch.randint(0, inputs.EMBED_ROWS, (60,), generator=g)])
    out = aq.aq_dequantize_rows(wq.to(DEV), sc.to(DEV), bi.to(DEV), group, bits, ids.to(DEV), dtype=out_dtype)
    aq.aq_device_error()
    got = out.cpu()
    got = got.view(torch.int32).numpy().view(np.uint32) if out_dtype == torch.float32 else half_bits(got)
    exp = _expected(wq, sc, bi, K, group, bits, ids.numpy(), sd, out_dtype)
    assert got.shape == (ids.numel(), K)
    assert np.array_equal(got, exp)


def test_rows_strided_output_and_canaries():
    """Rows land in a strided output; nothing outside it is written."""
    bits = 8
    wq, sc, bi, K, group = inputs.embedding_table(bits, rows=4096, seed=5)
    ids = torch.tensor([3, 4095, 0, 17], dtype=torch.int64)
    buf = torch.full((6, K + 64), 7.0, dtype=torch.bfloat16, device=DEV)
    out = buf[1:5, 32:32 + K]
    aq.aq_dequantize_rows(wq.to(DEV), sc.to(DEV), bi.to(DEV), group, bits, ids.to(DEV), out=out)
    b = buf.float().cpu()
    assert torch.all(b[0] == 7.0) and torch.all(b[5] == 7.0)
    assert torch.all(b[:, :32] == 7.0) and torch.all(b[:, 32 + K:] == 7.0)
    exp = _expected(wq, sc, bi, K, group, bits, ids.numpy(), "bf16", torch.bfloat16)
    assert np.array_equal(half_bits(out.cpu()), exp)


def test_rows_out_of_range_ids_flagged():
    """Ids outside the table give zero rows and AQ_ERR_INDEX from aq_device_error; the other rows
    are still exact, and the next call is clean."""
    bits = 4
    wq, sc, bi, K, group = inputs.embedding_table(bits, rows=1000, seed=6)
    ids = torch.tensor([5, -1, 999, 1000, 7], dtype=torch.int64)
    wqd, scd, bid = wq.to(DEV), sc.to(DEV), bi.to(DEV)
    out = aq.aq_dequantize_rows(wqd, scd, bid, group, bits, ids.to(DEV))
    with pytest.raises(aq.AQError) as ei:
        aq.aq_device_error()
    assert ei.value.name == "AQ_ERR_INDEX"
    got = out.float().cpu()
    assert torch.all(got[1] == 0) and torch.all(got[3] == 0)
    good = np.array([0, 2, 4])
    exp = _expected(wq, sc, bi, K, group, bits, ids.numpy()[good], "bf16", torch.bfloat16)
    assert np.array_equal(half_bits(out.cpu())[good], exp)
    aq.aq_dequantize_rows(wqd, scd, bid, group, bits, torch.tensor([1, 2], device=DEV))
    aq.aq_device_error()
