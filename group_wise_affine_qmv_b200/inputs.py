"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers and lays out shapes.  It holds none of
the method's arithmetic (no quantization, packing, dequantization or
contraction), so both the CUDA path and the CPU oracle can be fed from it
without sharing any of the computation.

Workloads (shapes and distributions from the pages and the method statement):

* probe -- transformers issue #47331, probe script: K=2048, N=1024, G=64,
  bits=4, ``torch.manual_seed(0)``, W ~ N(0,1) fp32 [N, K], x bf16 ~ N(0,1) in
  shapes [2, K], [2, 1, K], [2, 4, K].
* decode sweep -- projections of a 28-layer 0.6B-class decoder at a decode
  batch of 32 (x [32, 1, K]), W ~ N(0, 0.02), G=64, bits 4 and 8.
* ragged qmv -- bits 2/3/5/6, G 32/128, K=4096, N in {1,4,7,1001,4099},
  x [1, K] and [4, 1, K]; plus the running-sum stress case (mlx PR #4516:
  inputs whose half-precision partial sums round).
* strided views -- candle "Metal batched matmul" pitfall page: Q and K
  narrowed from a stacked qkv [2, 12, 5, 64]; a Linear on x narrowed from
  [2, 4, 3, 1408].
* prefill -- x [8, 2048, 4096] against W [14336, 4096] and the down
  projection x [8, 2048, 14336] against W [4096, 14336]; and a mixture-of-
  experts bank of 128 experts [2816, 1408] (8-bit, G=32; tensor shapes of the
  "Metal Kernel Bits=8 Final Report", section 4.3) with 256 tokens each routed
  to 8 distinct experts drawn uniformly.
"""
from __future__ import annotations

import torch

# ---------------------------------------------------------------------------
# generic draws
# ---------------------------------------------------------------------------


def gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float = 1.0, dtype=torch.float32, seed: int = 0, device: str = "cpu") -> torch.Tensor:
    """Seeded N(0, std^2) draw, generated in fp32 then cast to ``dtype``."""
    t = torch.randn(*shape, generator=gen(seed, device), dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


# ---------------------------------------------------------------------------
# probe (issue #47331 probe script)
# ---------------------------------------------------------------------------

PROBE = dict(K=2048, N=1024, group=64, bits=4)
PROBE_X_SHAPES = [(2, 2048), (2, 1, 2048), (2, 4, 2048)]


def probe_case():
    """W fp32 [1024, 2048] and the three x shapes, drawn in the page's order from seed 0."""
    torch.manual_seed(0)
    K, N = PROBE["K"], PROBE["N"]
    w = torch.randn(N, K)
    xs = [torch.randn(*shape, dtype=torch.float32).to(torch.bfloat16) for shape in PROBE_X_SHAPES]
    return w, xs


# ---------------------------------------------------------------------------
# decode sweep over a 0.6B-class decoder
# ---------------------------------------------------------------------------

DECODE_LAYERS = 28
DECODE_BATCH = 32
DECODE_GROUP = 64
# (name, K, N) per layer; "o" is the literal K=N=1024 reading, "o_alt" the 16x128-head one
DECODE_PROJ = [("q", 1024, 2048), ("k", 1024, 1024), ("v", 1024, 1024), ("o", 1024, 1024),
               ("gate", 1024, 3072), ("up", 1024, 3072), ("down", 3072, 1024)]
DECODE_PROJ_ALT_O = ("o_alt", 2048, 1024)
LM_HEAD = ("lm_head", 1024, 151936)
W_STD = 0.02


def decode_sweep_shapes(layers: int = DECODE_LAYERS):
    """List of (name, K, N) for every matrix of one decode step, lm_head last."""
    out = []
    for layer in range(layers):
        for name, K, N in DECODE_PROJ:
            out.append((f"L{layer}.{name}", K, N))
    out.append(LM_HEAD)
    return out


def decode_x(K: int, batch: int = DECODE_BATCH, seed: int = 1, device: str = "cpu") -> torch.Tensor:
    return normal((batch, 1, K), 1.0, torch.bfloat16, seed=seed, device=device)


def decode_w(K: int, N: int, seed: int, device: str = "cpu") -> torch.Tensor:
    return normal((N, K), W_STD, torch.float32, seed=seed, device=device)


# ---------------------------------------------------------------------------
# ragged-output qmv and the running-sum stress case
# ---------------------------------------------------------------------------

RAGGED_BITS = (2, 3, 5, 6)
RAGGED_GROUPS = (32, 128)
RAGGED_K = 4096
RAGGED_N = (1, 4, 7, 1001, 4099)
RAGGED_X_SHAPES = ((1, 4096), (4, 1, 4096))


def ragged_case(bits: int, group: int, N: int, x_shape, seed: int = 0):
    w = normal((N, RAGGED_K), 1.0, torch.float32, seed=seed)
    x = normal(x_shape, 1.0, torch.bfloat16, seed=seed + 1)
    return w, x


def stress_x(K: int, rows: int, dtype: torch.dtype) -> torch.Tensor:
    """Running-sum stress input: 1.0 and a small value interleaved.

    bf16 uses 2^-9 (the stated case: it rounds away against 1.0 once partial
    sums are formed in bf16).  fp16 uses 2^-12 so that chunk sums of 8 round in
    fp16 too (2^-9 would be exact there).  The exact sum of every 2-element
    pair is representable in fp32.
    """
    small = 2.0 ** -9 if dtype == torch.bfloat16 else 2.0 ** -12
    row = torch.empty(K, dtype=torch.float32)
    row[0::2] = 1.0
    row[1::2] = small
    return row.repeat(rows, 1).to(dtype)


def stress_w(N: int, K: int, value: float = 1.0) -> torch.Tensor:
    """Weights constant in every group, so the quantizer gives scale 0, q 0, bias = value."""
    return torch.full((N, K), value, dtype=torch.float32)


# ---------------------------------------------------------------------------
# strided batched views (candle pitfall page)
# ---------------------------------------------------------------------------


def qkv_case(seed: int = 3):
    """qkv [2, 12, 5, 64]; Q = narrow(1, 0, 4), K = narrow(1, 4, 4): strides [3840, 320, 64, 1]."""
    qkv = normal((2, 12, 5, 64), 1.0, torch.bfloat16, seed=seed)
    q = qkv.narrow(1, 0, 4)
    k = qkv.narrow(1, 4, 4)
    return qkv, q, k


def linear4d_case(seed: int = 4):
    """x = narrow(1, 0, 2) of [2, 4, 3, 1408] (strides [16896, 4224, 1408, 1]); W [2816, 1408]."""
    base = normal((2, 4, 3, 1408), 1.0, torch.bfloat16, seed=seed)
    x = base.narrow(1, 0, 2)
    w = normal((2816, 1408), W_STD, torch.float32, seed=seed + 1)
    return base, x, w


# ---------------------------------------------------------------------------
# quantized embedding table ("Metal Kernel Bits=8 Final Report", section 4.1)
# ---------------------------------------------------------------------------

EMBED_ROWS = 262144
EMBED_WORDS = 352          # uint32 words per row: K = 352 * 32 / bits
EMBED_GROUPS = 44          # scales per row: G = K / 44 (32 at 8 bits, 64 at 4 bits)


def embedding_table(bits: int, rows: int = EMBED_ROWS, sdtype=torch.bfloat16, seed: int = 0, device: str = "cpu"):
    """A packed table of random codes (uniform random uint32 words) with random scales
    (|N(0, 0.01)|) and biases (N(0, 0.05)) in the half dtype: (wq int32 [rows, 352],
    scales [rows, 44], biases [rows, 44], K, group)."""
    g = gen(seed, device)
    wq = torch.randint(-2 ** 31, 2 ** 31, (rows, EMBED_WORDS), generator=g, dtype=torch.int64,
                       device=device).to(torch.int32)
    sc = torch.randn(rows, EMBED_GROUPS, generator=g, device=device).abs_().mul_(0.01).to(sdtype)
    bi = torch.randn(rows, EMBED_GROUPS, generator=g, device=device).mul_(0.05).to(sdtype)
    K = EMBED_WORDS * 32 // bits
    return wq, sc, bi, K, K // EMBED_GROUPS


# ---------------------------------------------------------------------------
# prefill and the expert bank
# ---------------------------------------------------------------------------

PREFILL_X = (8, 2048, 4096)
PREFILL_W_UP = (14336, 4096)
PREFILL_X_DOWN = (8, 2048, 14336)
PREFILL_W_DOWN = (4096, 14336)
PREFILL_GROUP = 64

MOE_EXPERTS = 128
MOE_N = 2816
MOE_K = 1408
MOE_GROUP = 32
MOE_BITS = 8
MOE_TOKENS = 256
MOE_TOPK = 8


def moe_routing(tokens: int = MOE_TOKENS, experts: int = MOE_EXPERTS, topk: int = MOE_TOPK,
                seed: int = 0) -> torch.Tensor:
    """[tokens, topk] int64: each token's ``topk`` distinct experts, uniform at random."""
    g = gen(seed)
    return torch.stack([torch.randperm(experts, generator=g)[:topk] for _ in range(tokens)])


def moe_sort(routing: torch.Tensor, experts: int = MOE_EXPERTS):
    """Order the routed (token, expert) pairs by expert (stable in token order).

    Returns (token_index [T*topk] int64, offsets [experts+1] int64): rows
    offsets[e] .. offsets[e+1]-1 of the sorted activations belong to expert e.
    Pure index bookkeeping: no arithmetic of the method.
    """
    tok = torch.arange(routing.shape[0]).repeat_interleave(routing.shape[1])
    exp = routing.reshape(-1)
    order = torch.sort(exp * routing.shape[0] + tok).indices
    counts = torch.bincount(exp, minlength=experts)
    offsets = torch.zeros(experts + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    return tok[order], offsets
