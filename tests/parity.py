"""Comparison helpers for the GPU-vs-oracle parity tests (no arithmetic of the method)."""
import numpy as np
import torch

import oracle


def half_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16/f16 tensor (CPU copy, contiguous)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dtype_name(t: torch.Tensor) -> str:
    return {torch.bfloat16: "bf16", torch.float16: "f16"}[t.dtype]


def to_device_quant(Q, device="cuda", sdtype=torch.bfloat16):
    """Oracle quantization result -> (wq int32, scales, biases) device tensors (bit copies)."""
    wq = torch.from_numpy(Q.packed.view(np.int32).copy()).to(device)
    sc = torch.from_numpy(Q.scale_bits.view(np.int16).copy()).view(sdtype).to(device)
    bi = torch.from_numpy(Q.bias_bits.view(np.int16).copy()).view(sdtype).to(device)
    return wq, sc, bi


def oracle_linear_view(x: torch.Tensor, wdq: np.ndarray) -> np.ndarray:
    """Oracle contraction reading a CPU tensor x through its own strided view
    (storage offset and strides as they are, no contiguous copy)."""
    assert x.device.type == "cpu"
    xc = x.detach()
    base = xc.untyped_storage()
    flat = torch.empty(0, dtype=xc.dtype).set_(base, 0, (base.nbytes() // 2,), (1,))
    bits = flat.view(torch.int16).numpy().view(np.uint16)
    off = xc.storage_offset()
    shape = list(xc.shape)
    strides = list(xc.stride())
    if len(shape) == 1:
        shape, strides = [1] + shape, [shape[0]] + strides
    y = oracle.linear(bits[off:], dtype_name(xc), shape, strides, wdq)
    return y.reshape(tuple(x.shape[:-1]) + (wdq.shape[-2],))


def row_errors(y: torch.Tensor, ref: np.ndarray) -> np.ndarray:
    """Per-row max|y - ref| / max|ref| (the metric of transformers issue #47331's probe)."""
    yf = y.detach().float().cpu().double().numpy().reshape(-1, ref.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    num = np.abs(yf - r).max(-1)
    den = np.abs(r).max(-1)
    return num / np.maximum(den, 1e-300)


def assert_rows_close(y: torch.Tensor, ref: np.ndarray, x: torch.Tensor, wdq: np.ndarray, tol: float = 4e-3):
    """Every row within `tol` of the oracle by the page's per-row metric.

    Rows whose reference is dominated by cancellation (max|ref| below 1e-3 of
    the row's sum_k |x_k w_nk|, possible only for tiny N) are checked instead
    element by element against tol * sum_k |x_k w_nk|.
    """
    err = row_errors(y, ref)
    if np.all(err <= tol):
        return
    xf = np.abs(x.detach().float().cpu().double().numpy().reshape(-1, x.shape[-1]))
    mag = xf @ np.abs(wdq.reshape(-1, wdq.shape[-1])).T if wdq.ndim == 2 else None
    r = ref.reshape(-1, ref.shape[-1])
    yf = y.detach().float().cpu().double().numpy().reshape(-1, ref.shape[-1])
    for i in np.nonzero(err > tol)[0]:
        assert mag is not None and np.abs(r[i]).max() < 1e-3 * mag[i].max(), (i, err[i])
        assert np.all(np.abs(yf[i] - r[i]) <= tol * mag[i]), (i, err[i])
