"""Affine group-quantized linear layers for B200 (sm_100a).

``y = x . dequant(W)^T`` where W [N, K] is packed into uint32 words of
``bits``-wide codes q and every group of ``group`` consecutive K elements has
one half-precision scale and bias (``w = scale*q + bias``).

The compute lives in ``libaq.so`` (hand-written CUDA for sm_100a behind a C
ABI declared in ``include/aq.h``); ``aq`` is its thin ctypes binding.  Importing
this package does not load the library: ``aq`` loads it on first use and fails
loudly if it is missing or built for another device.
"""

__all__ = ["aq", "inputs"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
