"""CPU oracle for the affine group-quantized linear layer (test infrastructure).

This package is test infrastructure.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  The product path
(``group_wise_affine_qmv_b200``) never imports, links or executes anything here,
and this package never imports the product: the two share no code.

The arithmetic lives in ``aq_oracle.c`` (plain C, fp64 for every contraction,
IEEE fp32 for the quantizer's own steps).  This module only marshals numpy
arrays into it.  Function-level citations are in the C file; in short:

* ``quantize``    -- per-group min/max affine quantizer (transformers issue
  #47331, probe script: quantize fp32 W, then convert scales/biases to bf16).
* ``pack`` / ``unpack`` -- LSB-first little-endian bitstream per row.
* ``unpack_formula`` -- the packedIdx/shift/mask formula of "Metal Kernel
  Bits=8 Final Report" section 3.1 for 2/4/8 bits.
* ``dequant``     -- w' = s*q + b with the stored half-precision s, b, in fp64.
* ``linear``      -- y = x . w'^T in fp64, reading x through its strided view.
* ``linear_grouped`` -- the same per expert segment of a row-sorted x.
* ``silu`` / ``swiglu`` -- silu(g) * u in fp64 (the gated MLP step of the fused
  gate/up call).
* ``rms_inv`` -- 1 / sqrt(mean(x^2) + eps) per row (the normalised input option).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "aq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 1
F16 = 2

_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile aq_oracle.c into liboracle.so (gcc, no fast-math, no FMA contraction)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp = ctypes.c_void_p
            i64 = ctypes.c_int64
            ci = ctypes.c_int
            lib.oracle_quantize.argtypes = [vp, i64, i64, ci, ci, ci, vp, vp, vp, vp, vp]
            lib.oracle_quantize.restype = ci
            lib.oracle_pack.argtypes = [vp, i64, i64, ci, vp]
            lib.oracle_pack.restype = ci
            lib.oracle_unpack.argtypes = [vp, i64, i64, ci, vp]
            lib.oracle_unpack.restype = ci
            lib.oracle_unpack_formula.argtypes = [vp, i64, i64, ci, ci, vp]
            lib.oracle_unpack_formula.restype = ci
            lib.oracle_dequant.argtypes = [vp, vp, vp, ci, i64, i64, ci, vp]
            lib.oracle_dequant.restype = None
            lib.oracle_linear.argtypes = [vp, ci, ci, _i64p, _i64p, vp, ci, _i64p, _i64p, vp]
            lib.oracle_linear.restype = ci
            lib.oracle_linear_sampled.argtypes = [vp, ci, i64, i64, vp, i64, vp, vp, i64, vp]
            lib.oracle_linear_sampled.restype = None
            lib.oracle_linear_grouped.argtypes = [vp, ci, i64, i64, vp, i64, vp, i64, vp]
            lib.oracle_linear_grouped.restype = ci
            lib.oracle_factored_dot.argtypes = [vp, ci, vp, vp, vp, ci, i64, ci]
            lib.oracle_factored_dot.restype = ctypes.c_double
            lib.oracle_silu.argtypes = [ctypes.c_double]
            lib.oracle_silu.restype = ctypes.c_double
            lib.oracle_swiglu.argtypes = [vp, vp, i64, vp]
            lib.oracle_swiglu.restype = None
            lib.oracle_rms_inv.argtypes = [vp, ci, i64, i64, ctypes.c_double, vp]
            lib.oracle_rms_inv.restype = None
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16, ci]
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_float_to_half_rne.argtypes = [ctypes.c_float, ci]
            lib.oracle_float_to_half_rne.restype = ctypes.c_uint16
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _dtype_code(name: str) -> int:
    if name in ("bf16", "bfloat16"):
        return BF16
    if name in ("f16", "fp16", "float16"):
        return F16
    raise ValueError(f"half dtype expected, got {name}")


# --------------------------------------------------------------------------
# conversions
# --------------------------------------------------------------------------

def half_to_double(bits: np.ndarray, dtype: str) -> np.ndarray:
    lib = _load()
    code = _dtype_code(dtype)
    flat = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    out = np.array([lib.oracle_half_to_double(int(b), code) for b in flat], dtype=np.float64)
    return out.reshape(np.shape(bits))


def float_to_half_bits(values: np.ndarray, dtype: str) -> np.ndarray:
    lib = _load()
    code = _dtype_code(dtype)
    flat = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.array([lib.oracle_float_to_half_rne(float(v), code) for v in flat], dtype=np.uint16)
    return out.reshape(np.shape(values))


# --------------------------------------------------------------------------
# quantizer and packing
# --------------------------------------------------------------------------

class Quantized:
    """Oracle quantization result (all numpy)."""

    def __init__(self, codes, packed, scale32, bias32, scale_bits, bias_bits, group, bits, sdtype):
        self.codes = codes            # uint8 [..., N, K]
        self.packed = packed          # uint32 [..., N, K*bits/32]
        self.scale32 = scale32        # float32 [..., N, K/G]  (unrounded)
        self.bias32 = bias32          # float32 [..., N, K/G]
        self.scale_bits = scale_bits  # uint16 [..., N, K/G]   (stored half bits)
        self.bias_bits = bias_bits    # uint16 [..., N, K/G]
        self.group = group
        self.bits = bits
        self.sdtype = sdtype

    def dequant(self) -> np.ndarray:
        return dequant(self.codes, self.scale_bits, self.bias_bits, self.group, self.sdtype)


def quantize(w: np.ndarray, group: int, bits: int, sdtype: str = "bf16") -> Quantized:
    """Quantize fp32 W [..., N, K] group-wise; leading dims are treated as more rows."""
    lib = _load()
    w = np.ascontiguousarray(w, dtype=np.float32)
    if not np.all(np.isfinite(w)):
        raise ValueError("oracle quantize: W must be finite")
    shape = w.shape
    K = shape[-1]
    N = int(np.prod(shape[:-1]))
    if K % group != 0 or (K * bits) % 32 != 0:
        raise ValueError("K must be a multiple of the group and of 32/bits")
    ng = K // group
    codes = np.empty((N, K), np.uint8)
    scale32 = np.empty((N, ng), np.float32)
    bias32 = np.empty((N, ng), np.float32)
    sb = np.empty((N, ng), np.uint16)
    bb = np.empty((N, ng), np.uint16)
    rc = lib.oracle_quantize(_ptr(w), N, K, group, bits, _dtype_code(sdtype), _ptr(codes),
                             _ptr(scale32), _ptr(bias32), _ptr(sb), _ptr(bb))
    if rc != 0:
        raise ValueError("oracle_quantize rejected its arguments")
    packed = pack(codes, bits)
    lead = shape[:-1]
    return Quantized(codes.reshape(*lead, K), packed.reshape(*lead, K * bits // 32),
                     scale32.reshape(*lead, ng), bias32.reshape(*lead, ng),
                     sb.reshape(*lead, ng), bb.reshape(*lead, ng), group, bits, sdtype)


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    K = codes.shape[-1]
    N = int(np.prod(codes.shape[:-1]))
    out = np.empty((N, K * bits // 32), np.uint32)
    if lib.oracle_pack(_ptr(codes), N, K, bits, _ptr(out)) != 0:
        raise ValueError("K*bits must be a multiple of 32")
    return out.reshape(*codes.shape[:-1], K * bits // 32)


def unpack(packed: np.ndarray, K: int, bits: int) -> np.ndarray:
    lib = _load()
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    N = int(np.prod(packed.shape[:-1]))
    out = np.empty((N, K), np.uint8)
    if lib.oracle_unpack(_ptr(packed), N, K, bits, _ptr(out)) != 0:
        raise ValueError("K*bits must be a multiple of 32")
    return out.reshape(*packed.shape[:-1], K)


def unpack_formula(packed: np.ndarray, K: int, group: int, bits: int) -> np.ndarray:
    lib = _load()
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    N = int(np.prod(packed.shape[:-1]))
    out = np.empty((N, K), np.uint8)
    if lib.oracle_unpack_formula(_ptr(packed), N, K, group, bits, _ptr(out)) != 0:
        raise ValueError("formula form is defined for bits 2/4/8 only")
    return out.reshape(*packed.shape[:-1], K)


def dequant(codes: np.ndarray, scale_bits: np.ndarray, bias_bits: np.ndarray, group: int,
            sdtype: str = "bf16") -> np.ndarray:
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sb = np.ascontiguousarray(scale_bits, dtype=np.uint16)
    bb = np.ascontiguousarray(bias_bits, dtype=np.uint16)
    K = codes.shape[-1]
    N = int(np.prod(codes.shape[:-1]))
    out = np.empty((N, K), np.float64)
    lib.oracle_dequant(_ptr(codes), _ptr(sb), _ptr(bb), _dtype_code(sdtype), N, K, group, _ptr(out))
    return out.reshape(codes.shape)


# --------------------------------------------------------------------------
# contractions
# --------------------------------------------------------------------------

def linear(x_base: np.ndarray, x_dtype: str, x_shape, x_strides, wdq: np.ndarray) -> np.ndarray:
    """y = x . wdq^T in fp64.

    x_base: flat uint16 array holding the half bits of x's storage; x is the
    view (x_shape, x_strides) over it, strides in elements, offset 0.
    wdq: fp64 [..., N, K] (any leading batch dims broadcastable against x's).
    Returns fp64 of shape x_shape[:-1] + [N].
    """
    lib = _load()
    xb = np.ascontiguousarray(x_base, dtype=np.uint16).ravel()
    xs = np.array(list(x_shape), np.int64)
    xst = np.array(list(x_strides), np.int64)
    w = np.ascontiguousarray(wdq, dtype=np.float64)
    ws = np.array(w.shape, np.int64)
    wst = np.array([s // 8 for s in w.strides], np.int64)
    # bounds: the largest offset the view reaches must lie inside the buffer
    maxoff = int(sum((d - 1) * s for d, s in zip(xs, xst)))
    if maxoff >= xb.size or any(s < 0 for s in xst):
        raise ValueError("x view reaches outside its storage")
    out_shape = tuple(int(v) for v in xs[:-1]) + (int(ws[-2]),)
    y = np.empty(out_shape, np.float64)
    rc = lib.oracle_linear(_ptr(xb), _dtype_code(x_dtype), len(xs),
                           xs.ctypes.data_as(_i64p), xst.ctypes.data_as(_i64p),
                           _ptr(w), len(ws), ws.ctypes.data_as(_i64p), wst.ctypes.data_as(_i64p),
                           _ptr(y))
    if rc != 0:
        raise ValueError("oracle_linear rejected its arguments")
    return y


def linear_contig(x_bits: np.ndarray, x_dtype: str, wdq: np.ndarray) -> np.ndarray:
    """Convenience: x given as a contiguous uint16 array [..., K]."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    strides = [s // 2 for s in x_bits.strides]
    shape = list(x_bits.shape)
    if len(shape) == 1:
        shape = [1] + shape
        strides = [shape[-1]] + strides
    return linear(x_bits, x_dtype, shape, strides, wdq)


def linear_sampled(x_bits: np.ndarray, x_dtype: str, wdq: np.ndarray, rows, cols) -> np.ndarray:
    """fp64 outputs y[rows[i], cols[i]] for x [R, K] and wdq [N, K]."""
    lib = _load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w = np.ascontiguousarray(wdq, dtype=np.float64)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    c = np.ascontiguousarray(cols, dtype=np.int64)
    assert x.ndim == 2 and w.ndim == 2 and x.shape[1] == w.shape[1]
    assert r.shape == c.shape and (r.size == 0 or (r.max() < x.shape[0] and c.max() < w.shape[0]))
    out = np.empty(r.shape, np.float64)
    lib.oracle_linear_sampled(_ptr(x), _dtype_code(x_dtype), x.shape[1], x.shape[1], _ptr(w),
                              w.shape[1], _ptr(r), _ptr(c), r.size, _ptr(out))
    return out


def linear_grouped(x_bits: np.ndarray, x_dtype: str, offsets: np.ndarray, wdq_bank: np.ndarray) -> np.ndarray:
    """y[t] = x[t] . wdq_bank[e(t)]^T where rows offsets[e]..offsets[e+1]-1 belong to expert e."""
    lib = _load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    w = np.ascontiguousarray(wdq_bank, dtype=np.float64)
    T, K = x.shape
    E, N, K2 = w.shape
    assert K2 == K and off.size == E + 1
    y = np.empty((T, N), np.float64)
    if lib.oracle_linear_grouped(_ptr(x), _dtype_code(x_dtype), T, K, _ptr(off), E, _ptr(w), N, _ptr(y)) != 0:
        raise ValueError("bad expert offsets")
    return y


def factored_dot(x_bits: np.ndarray, x_dtype: str, codes: np.ndarray, scale_bits: np.ndarray,
                 bias_bits: np.ndarray, group: int, sdtype: str = "bf16") -> float:
    """One output row element in the factored s*sum(qx) + b*sum(x) form (fp64)."""
    lib = _load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    q = np.ascontiguousarray(codes, dtype=np.uint8)
    sb = np.ascontiguousarray(scale_bits, dtype=np.uint16)
    bb = np.ascontiguousarray(bias_bits, dtype=np.uint16)
    return lib.oracle_factored_dot(_ptr(x), _dtype_code(x_dtype), _ptr(q), _ptr(sb), _ptr(bb),
                                   _dtype_code(sdtype), x.shape[-1], group)


def silu(v: float) -> float:
    """silu(v) = v / (1 + exp(-v)) in fp64."""
    return _load().oracle_silu(float(v))


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """silu(g) * u elementwise, fp64 (g, u: fp64 results of the gate and up contractions)."""
    lib = _load()
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    assert g.shape == u.shape
    out = np.empty(g.shape, np.float64)
    lib.oracle_swiglu(_ptr(g), _ptr(u), g.size, _ptr(out))
    return out


def rms_inv(x_bits: np.ndarray, x_dtype: str, eps: float) -> np.ndarray:
    """1 / sqrt(mean_k x[t, k]^2 + eps) for every row of x [..., K] (half bits), fp64."""
    lib = _load()
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    K = x.shape[-1]
    rows = int(np.prod(x.shape[:-1]))
    out = np.empty(rows, np.float64)
    lib.oracle_rms_inv(_ptr(x), _dtype_code(x_dtype), rows, K, float(eps), _ptr(out))
    return out.reshape(x.shape[:-1])
