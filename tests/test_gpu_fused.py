"""GPU parity of the fused decode-layer calls (warp-level kernel) against the oracle, and of a
decode chain captured in a CUDA graph.

* aq_qmm_t_multi: up to three matrices sharing x (the q, k, v projections), one launch;
* aq_qmm_t_swiglu: silu(x . Wg^T) * (x . Wu^T), one launch;
* aq_qmm_t_residual: r + x . W^T, in place or into a separate y;
* a chain of decoder layers in which every call reads the previous call's output, launched as
  programmatic dependents inside one CUDA graph and replayed: checks that no kernel reads its
  input before the kernel that writes it has finished (the kernels prefetch weights before that
  wait, never activations).

The decoder layer the chain follows is the one of transformers issue #47331's reproduction (a
Qwen3-0.6B decoder, every projection a quantized linear on x [B, 1, hidden]): per layer
q, k, v = multi(norm(h)); h += o(v); a = swiglu(norm(h)); h += down(a); then lm_head(h), norm the
per-token RMS normalisation the fused calls apply to their input.  Attention itself is outside the
path: o reads v, which is what attention returns with a single cached position.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_qmv_b200 import aq, inputs
from tests.parity import dtype_name, half_bits, oracle_linear_view, row_errors, to_device_quant

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _q(w, group, bits, sdtype="bf16"):
    Q = oracle.quantize(w.float().numpy(), group, bits, sdtype)
    tdt = torch.bfloat16 if sdtype == "bf16" else torch.float16
    return Q, to_device_quant(Q, DEV, tdt)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("M,Ns,K", [(1, (100, 37, 64), 512), (5, (100, 37, 64), 512), (8, (2048, 1024, 1024), 1024),
                                    (32, (2048, 1024, 1024), 1024), (32, (33, 1, 300), 256), (16, (4099, 7), 4096)])
def test_multi_matches_oracle(bits, M, Ns, K):
    group = 64
    x = inputs.normal((M, 1, K), 1.0, torch.bfloat16, seed=M + K)
    xd = x.to(DEV)
    Qs, ws = [], []
    for j, N in enumerate(Ns):
        Q, w = _q(inputs.normal((N, K), 0.02, seed=100 * j + N + bits), group, bits)
        Qs.append(Q)
        ws.append(w)
    ys = aq.aq_qmm_t_multi(xd, ws, group, bits)
    for Q, y in zip(Qs, ys):
        err = row_errors(y, oracle_linear_view(x, Q.dequant()))
        assert err.size == M and np.all(err <= 4e-3), (err.max(), int(err.argmax()))


def test_multi_falls_back_to_plain_calls():
    """40 rows: the warp-level kernel does not take them, so each matrix runs as a plain call."""
    K, group, bits = 512, 64, 4
    x = inputs.normal((40, K), 1.0, torch.bfloat16, seed=3)
    Qs, ws = zip(*[_q(inputs.normal((N, K), 0.02, seed=N), group, bits) for N in (256, 130)])
    ys = aq.aq_qmm_t_multi(x.to(DEV), list(ws), group, bits)
    for Q, w, y in zip(Qs, ws, ys):
        assert np.all(row_errors(y, oracle_linear_view(x, Q.dequant())) <= 4e-3)
        assert torch.equal(y, aq.aq_qmm_t(x.to(DEV), *w, group, bits))


def test_multi_rejects_overlapping_outputs():
    K, group, bits = 256, 64, 4
    _, w = _q(inputs.normal((64, K), 0.02, seed=1), group, bits)
    x = torch.zeros(8, K, dtype=torch.bfloat16, device=DEV)
    buf = torch.empty(8, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(aq.AQError) as ei:
        aq.aq_qmm_t_multi(x, [w, w], group, bits, outs=[buf[:, :64], buf[:, 32:96]])
    assert ei.value.name == "AQ_ERR_OVERLAP"


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(1, 3072, 1024), (8, 1000, 1024), (32, 3072, 1024), (32, 17, 512),
                                   (13, 4099, 2048)])
def test_swiglu_matches_oracle(bits, M, N, K):
    group = 64
    x = inputs.normal((M, 1, K), 1.0, torch.bfloat16, seed=M * 3 + N)
    xd = x.to(DEV)
    Qg, wg = _q(inputs.normal((N, K), 0.02, seed=N + 1), group, bits)
    Qu, wu = _q(inputs.normal((N, K), 0.02, seed=N + 2), group, bits)
    y = aq.aq_qmm_t_swiglu(xd, wg, wu, group, bits)
    g = oracle_linear_view(x, Qg.dequant())
    u = oracle_linear_view(x, Qu.dequant())
    ref = oracle.swiglu(g, u)
    err = row_errors(y, ref)
    assert err.size == M and np.all(err <= 4e-3), (err.max(), int(err.argmax()))
    # fp32 output: the two contractions in fp32, the activation in fp32
    y32 = aq.aq_qmm_t_swiglu(xd, wg, wu, group, bits, out_dtype=torch.float32)
    assert np.all(row_errors(y32, ref) <= 1e-4)


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float16])
def test_swiglu_dtypes_and_groups(xdtype):
    M, N, K, bits = 24, 520, 2048, 4
    sd = dtype_name(torch.empty(0, dtype=xdtype))
    x = inputs.normal((M, K), 1.0, xdtype, seed=5)
    for group in (32, 64, 128):
        Qg, wg = _q(inputs.normal((N, K), 0.02, seed=group), group, bits, sd)
        Qu, wu = _q(inputs.normal((N, K), 0.02, seed=group + 1), group, bits, sd)
        y = aq.aq_qmm_t_swiglu(x.to(DEV), wg, wu, group, bits)
        ref = oracle.swiglu(oracle_linear_view(x, Qg.dequant()), oracle_linear_view(x, Qu.dequant()))
        assert np.all(row_errors(y, ref) <= 4e-3), group


RMS_EPS = 1e-6


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 8, 32])
def test_multi_and_swiglu_rms_normalised_input(bits, M):
    """The optional RMS-normalised input: every output of token t scaled by
    1 / sqrt(mean_k x[t,k]^2 + eps), before silu in the gate/up call."""
    K, group = 1024, 64
    x = inputs.normal((M, 1, K), 3.0, torch.bfloat16, seed=M + 90)
    xd = x.to(DEV)
    rinv = oracle.rms_inv(half_bits(x), "bf16", RMS_EPS).reshape(M, 1, 1)
    Qs, ws = zip(*[_q(inputs.normal((N, K), 0.02, seed=N + 91), group, bits) for N in (2048, 1024, 1024)])
    ys = aq.aq_qmm_t_multi(xd, list(ws), group, bits, rms_eps=RMS_EPS)
    for Q, y in zip(Qs, ys):
        ref = oracle_linear_view(x, Q.dequant()) * rinv
        assert np.all(row_errors(y, ref) <= 4e-3)
    Qg, wg = _q(inputs.normal((3072, K), 0.02, seed=92), group, bits)
    Qu, wu = _q(inputs.normal((3072, K), 0.02, seed=93), group, bits)
    y = aq.aq_qmm_t_swiglu(xd, wg, wu, group, bits, rms_eps=RMS_EPS)
    ref = oracle.swiglu(oracle_linear_view(x, Qg.dequant()) * rinv, oracle_linear_view(x, Qu.dequant()) * rinv)
    assert np.all(row_errors(y, ref) <= 4e-3)


def test_swiglu_unsupported_shape():
    K, group, bits = 512, 64, 4
    _, w = _q(inputs.normal((64, K), 0.02, seed=1), group, bits)
    x = torch.zeros(40, K, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(aq.AQError) as ei:
        aq.aq_qmm_t_swiglu(x, w, w, group, bits)
    assert ei.value.name == "AQ_ERR_UNSUPPORTED"


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 8, 32])
@pytest.mark.parametrize("inplace", [False, True])
def test_residual_matches_oracle(bits, M, inplace):
    K, N, group = 1024, 1024, 64
    x = inputs.normal((M, 1, K), 1.0, torch.bfloat16, seed=M + 7)
    r = inputs.normal((M, 1, N), 1.0, torch.bfloat16, seed=M + 8)
    Q, w = _q(inputs.normal((N, K), 0.02, seed=N + bits), group, bits)
    rd = r.to(DEV)
    if inplace:
        y = aq.aq_qmm_t_residual(x.to(DEV), *w, group, bits, r=rd, out=rd)
        assert y.data_ptr() == rd.data_ptr()
    else:
        y = aq.aq_qmm_t_residual(x.to(DEV), *w, group, bits, r=rd)
        assert torch.equal(rd.cpu(), r)
    ref = r.double().numpy() + oracle_linear_view(x, Q.dequant())
    assert np.all(row_errors(y, ref) <= 4e-3)


# ---------------------------------------------------------------------------
# the decode chain, graph-captured, against the oracle's own chain
# ---------------------------------------------------------------------------

def _bf16_round(v: np.ndarray) -> np.ndarray:
    """What the GPU stores for an fp64 value: the nearest bf16 (through fp32)."""
    bits = oracle.float_to_half_bits(v.astype(np.float32), "bf16")
    return oracle.half_to_double(bits, "bf16")


def _chain_setup(layers, bits, vocab, seed0=1000, logits_dtype=torch.bfloat16):
    B, group = inputs.DECODE_BATCH, inputs.DECODE_GROUP
    proj = {name: (K, N) for name, K, N in inputs.DECODE_PROJ}
    Q, W = {}, {}
    for l in range(layers):
        for i, name in enumerate(("q", "k", "v", "o", "gate", "up", "down")):
            K, N = proj[name]
            Q[l, name], W[l, name] = _q(inputs.decode_w(K, N, seed=seed0 * (l + 1) + i), group, bits)
    Q["lm"], W["lm"] = _q(inputs.decode_w(1024, vocab, seed=5), group, bits)
    h0 = inputs.decode_x(1024, seed=11)
    bufs = {"h0": h0.to(DEV), "h": torch.empty(B, 1, 1024, dtype=torch.bfloat16, device=DEV),
            "q": torch.empty(B, 1, 2048, dtype=torch.bfloat16, device=DEV),
            "k": torch.empty(B, 1, 1024, dtype=torch.bfloat16, device=DEV),
            "v": torch.empty(B, 1, 1024, dtype=torch.bfloat16, device=DEV),
            "a": torch.empty(B, 1, 3072, dtype=torch.bfloat16, device=DEV),
            "logits": torch.empty(B, 1, vocab, dtype=logits_dtype, device=DEV)}
    return Q, W, h0, bufs


def _chain_calls(W, bufs, layers, bits):
    """The launches of the chain, in order, as closures (q, k, v = multi(norm(h)); h += o(v);
    a = swiglu(norm(h)); h += down(a); ...; logits = lm_head(h)), norm the per-token RMS
    normalisation the fused calls apply."""
    group = inputs.DECODE_GROUP
    b = bufs
    calls = []
    for l in range(layers):
        src = b["h0"] if l == 0 else b["h"]
        calls.append(lambda l=l, src=src: aq.aq_qmm_t_multi(src, [W[l, "q"], W[l, "k"], W[l, "v"]], group, bits,
                                                            outs=[b["q"], b["k"], b["v"]], rms_eps=RMS_EPS))
        calls.append(lambda l=l, src=src: aq.aq_qmm_t_residual(b["v"], *W[l, "o"], group, bits, r=src, out=b["h"]))
        calls.append(lambda l=l: aq.aq_qmm_t_swiglu(b["h"], W[l, "gate"], W[l, "up"], group, bits, out=b["a"],
                                                    rms_eps=RMS_EPS))
        calls.append(lambda l=l: aq.aq_qmm_t_residual(b["a"], *W[l, "down"], group, bits, r=b["h"], out=b["h"]))
    calls.append(lambda: aq.aq_qmm_t(b["h"], *W["lm"], group, bits, out=b["logits"]))
    return calls


def _graph_replays(calls, bufs, n=3):
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for c in calls:
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for c in calls:
            c()
    out = []
    for _ in range(n):
        for k in ("h", "logits", "a", "v"):
            bufs[k].zero_()
        g.replay()
        torch.cuda.synchronize()
        out.append((bufs["logits"].clone(), bufs["h"].clone()))
    aq.aq_device_error()
    del g
    return out


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_chain_graph_matches_oracle(bits):
    """One chained decoder layer (four dependent launches) and lm_head, in one CUDA graph,
    against the oracle's own chain; logits in fp32.

    Why one layer: every stored activation is rounded to bf16 on both sides, and where the GPU's
    fp32 sums and the oracle's fp64 sums fall on either side of a rounding boundary the two
    chains carry values one bf16 step apart; each such step spreads through the next dense layer
    and flips more roundings.  Simulated on the CPU (fp32 sums in shuffled orders against fp64
    sums, these weights) the fp32 logits' per-row error is 1.1-1.8e-3 after one layer, 2.9-3.1e-3
    after two and 4.5-5.5e-3 after three (1-3 %, 8-16 %, 18-29 % of the hidden state a step
    apart): past the single-matmul bar from three layers on, at it from two.  Longer chains are
    checked for ordering, bit for bit, below.
    """
    layers, vocab = 1, 4096
    B = inputs.DECODE_BATCH
    Q, W, h0, bufs = _chain_setup(layers, bits, vocab, logits_dtype=torch.float32)
    results = _graph_replays(_chain_calls(W, bufs, layers, bits), bufs)
    for r_ in results[1:]:
        assert torch.equal(r_[0], results[0][0]) and torch.equal(r_[1], results[0][1])

    # the oracle's chain: fp64 contractions, every stored activation rounded to bf16 as the GPU does
    def lin(xv, Qk):
        xb = half_bits(torch.from_numpy(xv.astype(np.float32)).to(torch.bfloat16)).reshape(B, -1)
        return oracle.linear_contig(xb, "bf16", Qk.dequant())

    def rinv(xv):
        xb = half_bits(torch.from_numpy(xv.astype(np.float32)).to(torch.bfloat16)).reshape(B, -1)
        return oracle.rms_inv(xb, "bf16", RMS_EPS)[:, None]

    hv = h0.reshape(B, 1024).double().numpy()
    for l in range(layers):
        vv = _bf16_round(lin(hv, Q[l, "v"]) * rinv(hv))
        hv = _bf16_round(hv + lin(vv, Q[l, "o"]))
        r = rinv(hv)
        av = _bf16_round(oracle.swiglu(lin(hv, Q[l, "gate"]) * r, lin(hv, Q[l, "up"]) * r))
        hv = _bf16_round(hv + lin(av, Q[l, "down"]))
    ref = lin(hv, Q["lm"])
    logits, h_out = results[-1]
    err = row_errors(logits, ref)
    assert err.size == B and np.all(err <= 4e-3), (err.max(), int(err.argmax()))
    # the residual stream, element by element: within two bf16 steps of the oracle's value (one
    # where the first residual's sums straddled a rounding boundary, one more where the second
    # did) plus one bf16 step of the row's largest value (an input element one step apart moves a
    # small output by an amount set by the inputs' scale, not by its own; a CPU simulation with
    # shuffled fp32 sums used up to 0.8 of half that)
    got = h_out.reshape(B, 1024).double().cpu().numpy()
    step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(hv), 2.0 ** -126))) - 7)
    row_scale = np.abs(hv).max(-1, keepdims=True)
    assert np.all(np.abs(got - hv) <= 2 * step + 2.0 ** -8 * row_scale)


def test_decode_chain_ordering_bitwise():
    """The full 28-layer chain (112 launches + lm_head), replayed from a CUDA graph in which every
    launch is a programmatic dependent of the one before, gives exactly the bits of the same calls
    run one at a time with the device drained after each: no kernel read an activation before the
    kernel that writes it had finished, and none wrote one that an earlier kernel still read."""
    layers, bits, vocab = inputs.DECODE_LAYERS, 4, 2048
    _, W, _, bufs = _chain_setup(layers, bits, vocab, seed0=7)
    calls = _chain_calls(W, bufs, layers, bits)
    results = _graph_replays(calls, bufs, n=2)
    for k in ("h", "logits", "a", "v"):
        bufs[k].zero_()
    for c in calls:
        c()
        torch.cuda.synchronize()
    assert torch.equal(bufs["logits"], results[0][0]) and torch.equal(bufs["h"], results[0][1])
    assert torch.equal(results[1][0], results[0][0])
