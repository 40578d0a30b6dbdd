"""Thin ctypes binding of libaq (include/aq.h): argument marshalling only.

Every function here turns torch tensors into ``aq_view`` descriptors, passes
the current CUDA stream, calls the C entry point of the same name and raises
``AQError`` on a non-OK status.  No arithmetic of the method happens in Python,
and there is no fallback: if ``libaq.so`` is missing or cannot be loaded, the
first call raises.

    wq, s, b = aq_quantize(w, group=64, bits=4)          # w [N, K] on cuda
    y = aq_qmm_t(x, wq, s, b, group=64, bits=4)            # x [..., K]
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libaq.so")

AQ_F32, AQ_BF16, AQ_F16, AQ_U32 = 0, 1, 2, 3
AQ_REGIME_QMV, AQ_REGIME_MMA = 0, 1
KERNEL_NAMES = {0: "gemv", 1: "warp_mma", 2: "tc_small_m", 3: "tc_prefill"}

_DT = {torch.float32: AQ_F32, torch.bfloat16: AQ_BF16, torch.float16: AQ_F16, torch.int32: AQ_U32,
       torch.uint32: AQ_U32}


class AQError(RuntimeError):
    def __init__(self, status: int, name: str, detail: str):
        super().__init__(f"{name}: {detail}" if detail else name)
        self.status = status
        self.name = name


class AqView(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class AqPlan(ctypes.Structure):
    _fields_ = [("regime", ctypes.c_int32), ("w_batched", ctypes.c_int32), ("M", ctypes.c_int64),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("nbatch_dims", ctypes.c_int32),
                ("kernel", ctypes.c_int32), ("batch_shape", ctypes.c_int64 * 2),
                ("x_batch_stride", ctypes.c_int64 * 2), ("y_batch_stride", ctypes.c_int64 * 2),
                ("w_batch_stride", ctypes.c_int64 * 2), ("s_batch_stride", ctypes.c_int64 * 2),
                ("b_batch_stride", ctypes.c_int64 * 2), ("x_row_stride", ctypes.c_int64),
                ("y_row_stride", ctypes.c_int64), ("total_rows", ctypes.c_int64), ("y_tiles", ctypes.c_int32)]


EXPORTED = ("aq_quantize", "aq_dequantize", "aq_dequantize_rows", "aq_qmv", "aq_qmm_t", "aq_qmm_t_grouped", "aq_qmv_gathered", "aq_qmm_t_multi",
            "aq_qmm_t_swiglu", "aq_qmm_t_residual", "aq_plan_linear", "aq_status_string", "aq_last_error_message",
            "aq_device_error", "aq_check_bounded_wait", "aq_version")

_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH):
    """Load libaq.so (once).  Raises if it is missing: there is no fallback path."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(f"libaq.so not built at {path}; run `python -m group_wise_affine_qmv_b200.build`")
        lib = ctypes.CDLL(path)
        V = ctypes.POINTER(AqView)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        for name in ("aq_qmv", "aq_qmm_t"):
            f = getattr(lib, name)
            f.argtypes = [V, V, V, V, ci, ci, V, vp]
            f.restype = ci
        lib.aq_quantize.argtypes = [V, ci, ci, V, V, V, vp]
        lib.aq_quantize.restype = ci
        lib.aq_dequantize.argtypes = [V, V, V, ci, ci, V, vp]
        lib.aq_dequantize.restype = ci
        lib.aq_dequantize_rows.argtypes = [V, V, V, ci, ci, vp, ctypes.c_int64, V, vp]
        lib.aq_dequantize_rows.restype = ci
        lib.aq_qmm_t_grouped.argtypes = [V, vp, ci, V, V, V, ci, ci, V, vp]
        lib.aq_qmm_t_grouped.restype = ci
        lib.aq_qmv_gathered.argtypes = [V, vp, vp, ctypes.c_int64, V, V, V, ci, ci, V, vp]
        lib.aq_qmv_gathered.restype = ci
        VA = ctypes.POINTER(V)
        lib.aq_qmm_t_multi.argtypes = [V, ci, VA, VA, VA, ci, ci, ctypes.c_float, VA, vp]
        lib.aq_qmm_t_multi.restype = ci
        lib.aq_qmm_t_swiglu.argtypes = [V, V, V, V, V, V, V, ci, ci, ctypes.c_float, V, vp]
        lib.aq_qmm_t_swiglu.restype = ci
        lib.aq_qmm_t_residual.argtypes = [V, V, V, V, ci, ci, V, V, vp]
        lib.aq_qmm_t_residual.restype = ci
        lib.aq_plan_linear.argtypes = [V, V, V, V, ci, ci, V, ci, ctypes.POINTER(AqPlan)]
        lib.aq_plan_linear.restype = ci
        lib.aq_status_string.argtypes = [ci]
        lib.aq_status_string.restype = ctypes.c_char_p
        lib.aq_last_error_message.argtypes = []
        lib.aq_last_error_message.restype = ctypes.c_char_p
        lib.aq_device_error.argtypes = [vp]
        lib.aq_device_error.restype = ci
        lib.aq_check_bounded_wait.argtypes = [ctypes.c_uint64, vp]
        lib.aq_check_bounded_wait.restype = ci
        lib.aq_version.argtypes = []
        lib.aq_version.restype = ci
        _lib = lib
        return lib


def view(t: torch.Tensor) -> AqView:
    """aq_view of a tensor (no copy; strides in elements)."""
    if t.dim() > 4 or t.dim() < 1:
        raise ValueError("aq views have rank 1..4")
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}")
    v = AqView()
    v.data = t.data_ptr() if t.numel() > 0 else (t.data_ptr() or None)
    v.dtype = _DT[t.dtype]
    v.rank = t.dim()
    for i in range(t.dim()):
        v.shape[i] = t.shape[i]
        v.stride[i] = t.stride(i)
    return v


def _stream(t: torch.Tensor) -> int:
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    return torch.cuda.current_stream(t.device).cuda_stream


def _check(lib, status: int):
    if status != 0:
        name = lib.aq_status_string(status).decode()
        detail = lib.aq_last_error_message().decode()
        raise AQError(status, name, detail)


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def aq_quantize(w: torch.Tensor, group: int, bits: int, scale_dtype: torch.dtype | None = None, out=None):
    """Group-wise affine quantization of w [N, K] -> (wq uint32 [N, K*bits/32], scales, biases),
    into ``out`` = (wq, scales, biases) when given."""
    lib = load_library()
    if scale_dtype is None:
        scale_dtype = w.dtype if w.dtype in (torch.bfloat16, torch.float16) else torch.bfloat16
    N, K = w.shape
    if out is not None:
        wq, sc, bi = out
    else:
        wq = torch.empty((N, K * bits // 32), dtype=torch.int32, device=w.device)
        sc = torch.empty((N, K // group), dtype=scale_dtype, device=w.device)
        bi = torch.empty((N, K // group), dtype=scale_dtype, device=w.device)
    with torch.cuda.device(w.device):
        _check(lib, lib.aq_quantize(view(w), group, bits, view(wq), view(sc), view(bi), _stream(w)))
    return wq, sc, bi


def aq_dequantize(wq, scales, biases, group: int, bits: int, dtype: torch.dtype = torch.float32):
    lib = load_library()
    N = wq.shape[0]
    K = wq.shape[1] * 32 // bits
    out = torch.empty((N, K), dtype=dtype, device=wq.device)
    with torch.cuda.device(wq.device):
        _check(lib, lib.aq_dequantize(view(wq), view(scales), view(biases), group, bits, view(out), _stream(wq)))
    return out


def aq_dequantize_rows(wq, scales, biases, group: int, bits: int, ids, dtype: torch.dtype = torch.bfloat16,
                       out=None):
    """Rows ids of the quantized table, dequantized: out [len(ids), K] (ids: int64 CUDA tensor)."""
    lib = load_library()
    if ids.dtype != torch.int64 or not ids.is_cuda or ids.dim() != 1 or not ids.is_contiguous():
        raise TypeError("ids must be a contiguous 1D int64 CUDA tensor")
    K = wq.shape[1] * 32 // bits
    if out is None:
        out = torch.empty((ids.numel(), K), dtype=dtype, device=wq.device)
    with torch.cuda.device(wq.device):
        _check(lib, lib.aq_dequantize_rows(view(wq), view(scales), view(biases), group, bits,
                                           ctypes.c_void_p(ids.data_ptr()), ids.numel(), view(out), _stream(wq)))
    return out


def _linear(fn: str, x, wq, scales, biases, group, bits, out=None, out_dtype=None):
    lib = load_library()
    N = wq.shape[-2]
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=out_dtype or x.dtype, device=x.device)
    with torch.cuda.device(x.device):
        _check(lib, getattr(lib, fn)(view(x), view(wq), view(scales), view(biases), group, bits, view(out),
                                     _stream(x)))
    return out


def aq_qmm_t(x, wq, scales, biases, group: int, bits: int, out=None, out_dtype=None):
    """y = x . dequant(W)^T; kernel chosen by rows per launch."""
    return _linear("aq_qmm_t", x, wq, scales, biases, group, bits, out, out_dtype)


def aq_qmv(x, wq, scales, biases, group: int, bits: int, out=None, out_dtype=None):
    """Same as aq_qmm_t but always the CUDA-core GEMV kernel."""
    return _linear("aq_qmv", x, wq, scales, biases, group, bits, out, out_dtype)


def aq_qmm_t_grouped(x_sorted, offsets, wq_bank, s_bank, b_bank, group: int, bits: int, out=None,
                     out_dtype=None):
    """Mixture-of-experts bank: rows offsets[e]..offsets[e+1]-1 of x_sorted use expert e."""
    lib = load_library()
    T = x_sorted.shape[0]
    N = wq_bank.shape[1]
    if offsets.dtype != torch.int64 or not offsets.is_cuda:
        raise TypeError("offsets must be an int64 CUDA tensor")
    if out is None:
        out = torch.empty((T, N), dtype=out_dtype or x_sorted.dtype, device=x_sorted.device)
    with torch.cuda.device(x_sorted.device):
        _check(lib, lib.aq_qmm_t_grouped(view(x_sorted), ctypes.c_void_p(offsets.data_ptr()), wq_bank.shape[0],
                                         view(wq_bank), view(s_bank), view(b_bank), group, bits, view(out),
                                         _stream(x_sorted)))
    return out


def aq_qmm_t_multi(x, weights, group: int, bits: int, outs=None, out_dtype=None, rms_eps: float = 0.0):
    """y[j] = x . dequant(W_j)^T for up to three (wq, scales, biases) sharing x, in one launch
    where the warp-level kernel takes them (rms_eps > 0: x RMS-normalised per token first).
    Returns the list of outputs."""
    lib = load_library()
    n = len(weights)
    if outs is None:
        outs = [torch.empty(tuple(x.shape[:-1]) + (w[0].shape[-2],), dtype=out_dtype or x.dtype, device=x.device)
                for w in weights]
    V = ctypes.POINTER(AqView)
    keep = [[view(w[i]) for w in weights] for i in range(3)] + [[view(o) for o in outs]]
    arrs = [(V * n)(*[ctypes.pointer(v) for v in vs]) for vs in keep]
    with torch.cuda.device(x.device):
        _check(lib, lib.aq_qmm_t_multi(view(x), n, arrs[0], arrs[1], arrs[2], group, bits, float(rms_eps), arrs[3],
                                       _stream(x)))
    return outs


def aq_qmm_t_swiglu(x, gate, up, group: int, bits: int, out=None, out_dtype=None, rms_eps: float = 0.0):
    """y = silu(x . dequant(W_gate)^T) * (x . dequant(W_up)^T); gate, up = (wq, scales, biases);
    rms_eps > 0: x RMS-normalised per token first."""
    lib = load_library()
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (gate[0].shape[-2],), dtype=out_dtype or x.dtype, device=x.device)
    with torch.cuda.device(x.device):
        _check(lib, lib.aq_qmm_t_swiglu(view(x), view(gate[0]), view(gate[1]), view(gate[2]), view(up[0]),
                                        view(up[1]), view(up[2]), group, bits, float(rms_eps), view(out),
                                        _stream(x)))
    return out


def aq_qmm_t_residual(x, wq, scales, biases, group: int, bits: int, r, out=None):
    """y = r + x . dequant(W)^T (out may be r itself: an in-place residual update)."""
    lib = load_library()
    if out is None:
        out = torch.empty_like(r)
    with torch.cuda.device(x.device):
        _check(lib, lib.aq_qmm_t_residual(view(x), view(wq), view(scales), view(biases), group, bits, view(r),
                                          view(out), _stream(x)))
    return out


def aq_qmv_gathered(x, x_ids, w_ids, wq_bank, s_bank, b_bank, group: int, bits: int, out=None, out_dtype=None):
    """y[i] = x[x_ids[i]] . dequant(W[w_ids[i]])^T (ids: contiguous 1D int64 CUDA tensors)."""
    lib = load_library()
    for ids in (x_ids, w_ids):
        if ids.dtype != torch.int64 or not ids.is_cuda or ids.dim() != 1 or not ids.is_contiguous():
            raise TypeError("ids must be contiguous 1D int64 CUDA tensors")
    if x_ids.numel() != w_ids.numel():
        raise ValueError("x_ids and w_ids must have the same length")
    R = x_ids.numel()
    if out is None:
        out = torch.empty((R, wq_bank.shape[1]), dtype=out_dtype or x.dtype, device=x.device)
    with torch.cuda.device(x.device):
        _check(lib, lib.aq_qmv_gathered(view(x), ctypes.c_void_p(x_ids.data_ptr()), ctypes.c_void_p(w_ids.data_ptr()),
                                        R, view(wq_bank), view(s_bank), view(b_bank), group, bits, view(out),
                                        _stream(x)))
    return out


def aq_plan_linear(x, wq, scales, biases, group: int, bits: int, y, force_qmv: bool = False) -> dict:
    """Host-only: how aq_qmm_t (or aq_qmv) would run this call.  Tensors may live on the CPU."""
    lib = load_library()
    p = AqPlan()
    _check(lib, lib.aq_plan_linear(view(x), view(wq), view(scales), view(biases), group, bits, view(y),
                                   1 if force_qmv else 0, ctypes.byref(p)))
    note = lib.aq_last_error_message().decode()
    return dict(regime="mma" if p.regime == AQ_REGIME_MMA else "qmv", kernel=KERNEL_NAMES[p.kernel],
                w_batched=bool(p.w_batched), M=p.M, N=p.N,
                K=p.K, nbatch_dims=p.nbatch_dims, batch_shape=tuple(p.batch_shape),
                x_batch_stride=tuple(p.x_batch_stride), y_batch_stride=tuple(p.y_batch_stride),
                w_batch_stride=tuple(p.w_batch_stride), x_row_stride=p.x_row_stride, y_row_stride=p.y_row_stride,
                total_rows=p.total_rows, y_tiles=bool(p.y_tiles), note=note)


def aq_device_error(device=None):
    """Synchronize the current stream and read/clear the device-side error word."""
    lib = load_library()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib, lib.aq_device_error(torch.cuda.current_stream(dev).cuda_stream))


def aq_check_bounded_wait(budget_ns: int, device=None):
    """Enqueue the bounded-wait self-check (a wait on a barrier nothing completes, given up after
    budget_ns); the next aq_device_error() then raises AQ_ERR_TIMEOUT."""
    lib = load_library()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib, lib.aq_check_bounded_wait(int(budget_ns), torch.cuda.current_stream(dev).cuda_stream))


def aq_version() -> int:
    return load_library().aq_version()
