#!/usr/bin/env python3
"""Benchmark: the decode step of a 28-layer 0.6B-class decoder through libaq.

One step = for 4-bit AND 8-bit weights (G = 64), a chain of 28 decoder layers at a
decode batch of 32 tokens followed by lm_head, every call reading the previous call's
output (the decoder layer of transformers issue #47331's reproduction, attention left
out: o reads v, which is what attention returns with one cached position):

    q, k, v = aq_qmm_t_multi(h, [Wq, Wk, Wv])    h += aq_qmm_t_residual(v, Wo)
    a = aq_qmm_t_swiglu(h, Wgate, Wup)           h += aq_qmm_t_residual(a, Wdown)
    logits = aq_qmm_t(h, Wlm_head)

All weights are distinct and resident in HBM (1.07 GB per step, larger than L2, so
every step streams its weights from HBM).  The step is captured once in a CUDA graph
(every tensor-core kernel a programmatic dependent of the one before) and replayed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  `value` is whole-job HBM throughput in GB/s
(algorithmic bytes: packed W + scales + biases + every activation read or written,
each counted once per launch) with inputs resident on the device; `e2e` is the same
metric with the step's input hidden state copied host->device and the logits copied
back inside the timed region.  Multi-GPU runs are independent replicas (the operation
has no exchange step on one layer): per-GPU work is fixed.  The reference arm
(--impl reference) times the CPU oracle on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from group_wise_affine_qmv_b200 import inputs  # noqa: E402

METRIC = "W4/W8 qmm_t µs and HBM GB/s (% of peak) decode; prefill TFLOP/s (% bf16 peak)"
GROUP = inputs.DECODE_GROUP
BITS_LIST = (4, 8)
FALLBACK_HBM_GBS = 6650.0


def w_bytes(K, N, bits):
    """Packed W + bf16 scales + bf16 biases of one matrix."""
    return N * K * bits // 8 + 2 * 2 * N * (K // GROUP)


def matrix_bytes(K, N, bits, M=inputs.DECODE_BATCH):
    """Algorithmic bytes of one plain call: W + scales + biases + x + y (bf16)."""
    return w_bytes(K, N, bits) + 2 * M * K + 2 * M * N


def sweep_shapes(layers):
    return inputs.decode_sweep_shapes(layers)


def sweep_bytes(layers):
    """Bytes of the unfused sweep: every matrix of the step as its own call on a fixed x."""
    tot = 0
    for bits in BITS_LIST:
        for _, K, N in sweep_shapes(layers):
            tot += matrix_bytes(K, N, bits)
    return tot


PROJ = {name: (K, N) for name, K, N in inputs.DECODE_PROJ}
RMS_EPS = 1e-6   # the block inputs' RMS normalisation, fused into the q/k/v and gate/up calls
HIDDEN = PROJ["q"][0]


def layer_launch_bytes(bits, M=inputs.DECODE_BATCH):
    """Algorithmic bytes of the four launches of one chained decoder layer, in order:
    multi(q,k,v): 3 W + h + q,k,v;  residual(o): W + v + h (read) + h (write);
    swiglu: 2 W + h + a;  residual(down): W + a + h + h."""
    a = lambda n: 2 * M * n   # one bf16 activation row set of width n
    q, k, v, o, g, u, d = (PROJ[n] for n in ("q", "k", "v", "o", "gate", "up", "down"))
    return [w_bytes(*q, bits) + w_bytes(*k, bits) + w_bytes(*v, bits) + a(HIDDEN) + a(q[1]) + a(k[1]) + a(v[1]),
            w_bytes(*o, bits) + a(o[0]) + 2 * a(o[1]),
            w_bytes(*g, bits) + w_bytes(*u, bits) + a(HIDDEN) + a(g[1]),
            w_bytes(*d, bits) + a(d[0]) + 2 * a(d[1])]


def chain_bytes(layers, bits):
    K, N = inputs.LM_HEAD[1], inputs.LM_HEAD[2]
    return layers * sum(layer_launch_bytes(bits)) + matrix_bytes(K, N, bits)


def step_bytes(layers):
    return sum(chain_bytes(layers, bits) for bits in BITS_LIST)


def bench_config(layers, world):
    """The workload this benchmark's lines are quoted on (both arms)."""
    return {"workload": "decode step: 28 chained decoder layers (fused q/k/v, o + residual, fused gate/up + "
                        "silu*mul, down + residual) + lm_head, x [32,1,1024] bf16, bits 4 and 8, G=64",
            "tokens": inputs.DECODE_BATCH, "layers": layers, "bits": list(BITS_LIST), "group": GROUP,
            "bytes_per_step": step_bytes(layers), "launches_per_step": len(BITS_LIST) * (4 * layers + 1),
            "l2": "inputs larger than L2 (weights streamed from HBM each step)",
            "graph": "one CUDA graph per step, programmatic dependent launches", "parallelism": f"replicas x{world}"}


def bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except Exception:
        return 1590.0, "fallback"


def time_calls(fn, reps, stream):
    """Average device time (ms) of `fn` over `reps` calls on `stream` (CUDA events)."""
    with torch.cuda.stream(stream):
        fn()
        fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def _l2_bytes(device):
    try:
        return torch.cuda.get_device_properties(device).L2_cache_size
    except Exception:
        return 126 * 1024 * 1024


def probe_and_ragged(device, stream):
    """Configs 1 and 3 with cold weights: each shape's quantized W is copied until the copies
    exceed twice the L2 size, and one CUDA graph calls the shape once per copy, so every call
    streams its weights from HBM (reported per call: the probe, K 2048, N 1024, 4-bit G64, x [2,K],
    [2,1,K], [2,4,K]; the ragged GEMV, K 4096, N 1001 / 4099, bits 2/3/5/6, G 32/128, x [1,K] and
    [4,1,K])."""
    from group_wise_affine_qmv_b200 import aq
    hbm, _ = hbm_peak()
    l2 = _l2_bytes(device)
    out = {"l2_condition": f"weights rotated over copies totalling > 2 x L2 ({l2 // 2**20} MiB): HBM-cold calls"}

    def rotated(fn_call, w3, nbytes_w, calls_cap=400):
        n = min(calls_cap, max(2, -(-2 * l2 // nbytes_w)))
        copies = [tuple(t_.clone() for t_ in w3) for _ in range(n)]
        g = graph_of(lambda: [fn_call(*c) for c in copies], stream)
        ms = time_graph(g, 5, stream)
        del g, copies
        return ms / n, n

    w, xs = inputs.probe_case()
    wq, sc, bi = aq.aq_quantize(w.to(device), 64, 4, scale_dtype=torch.bfloat16)
    wbytes = wq.numel() * 4 + sc.numel() * 4
    for x in xs:
        xd = x.to(device)
        ms, n = rotated(lambda a, b_, c: aq.aq_qmm_t(xd, a, b_, c, 64, 4), (wq, sc, bi), wbytes)
        M = x.numel() // x.shape[-1]
        nbytes = wbytes + 2 * M * (2048 + 1024)
        out["probe_x" + "x".join(str(d) for d in x.shape)] = {"us": round(ms * 1e3, 2), "copies": n,
                                                              "GBps": round(nbytes / ms / 1e6, 1),
                                                              "frac_of_hbm_peak": round(nbytes / ms / 1e6 / hbm, 4)}
    for bits in (2, 3, 5, 6):
        for group in (32, 128):
            for N in (1001, 4099):
                w, _ = inputs.ragged_case(bits, group, N, (1, inputs.RAGGED_K))
                wq, sc, bi = aq.aq_quantize(w.to(device), group, bits, scale_dtype=torch.bfloat16)
                wbytes = wq.numel() * 4 + sc.numel() * 4
                for shape in ((1, inputs.RAGGED_K), (4, 1, inputs.RAGGED_K)):
                    x = inputs.normal(shape, 1.0, torch.bfloat16, seed=3, device=device)
                    ms, n = rotated(lambda a, b_, c: aq.aq_qmv(x, a, b_, c, group, bits), (wq, sc, bi), wbytes)
                    M = 1 if len(shape) == 2 else 4
                    nbytes = wbytes + 2 * M * (inputs.RAGGED_K + N)
                    out[f"qmv_b{bits}_g{group}_n{N}_m{M}"] = {"us": round(ms * 1e3, 2), "copies": n,
                                                            "GBps": round(nbytes / ms / 1e6, 1),
                                                            "frac_of_hbm_peak": round(nbytes / ms / 1e6 / hbm, 4)}
    return out


def prefill_and_moe(device, stream):
    """Config 5: the decoder MLP's prefill shapes (x [8,2048,K] bf16, W 4- and 8-bit, G=64) and
    the mixture-of-experts bank (128 experts [2816, 1408], 8-bit, G=32, 256 tokens routed top-8),
    each call timed alone with CUDA events; inputs synthetic and generated on the device."""
    from group_wise_affine_qmv_b200 import aq
    peak, peak_kind = bf16_peak()
    out = {"peak_tflops": peak, "peak_source": peak_kind}
    for tag, xs, (N, K) in (("up", inputs.PREFILL_X, inputs.PREFILL_W_UP),
                            ("down", inputs.PREFILL_X_DOWN, inputs.PREFILL_W_DOWN)):
        x = inputs.normal(xs, 1.0, torch.bfloat16, seed=5, device=device)
        M = xs[0] * xs[1]
        for bits in BITS_LIST:
            w = inputs.normal((N, K), inputs.W_STD, seed=6 + bits, device=device)
            wq, sc, bi = aq.aq_quantize(w, inputs.PREFILL_GROUP, bits, scale_dtype=torch.bfloat16)
            del w
            y = torch.empty(xs[:-1] + (N,), dtype=torch.bfloat16, device=device)
            ms = time_calls(lambda: aq.aq_qmm_t(x, wq, sc, bi, inputs.PREFILL_GROUP, bits, out=y), 5, stream)
            tf = 2.0 * M * N * K / ms / 1e9
            out[f"{tag}_w{bits}"] = {"x": list(xs), "W": [N, K], "ms": round(ms, 3), "TFLOPs": round(tf, 1),
                                    "frac_of_peak": round(tf / peak, 4)}
            del wq, sc, bi, y
        del x
    # expert bank
    E, N, K, G, bits = inputs.MOE_EXPERTS, inputs.MOE_N, inputs.MOE_K, inputs.MOE_GROUP, inputs.MOE_BITS
    wq = torch.empty(E, N, K * bits // 32, dtype=torch.int32, device=device)
    sc = torch.empty(E, N, K // G, dtype=torch.bfloat16, device=device)
    bi = torch.empty_like(sc)
    for e in range(E):
        w = inputs.normal((N, K), inputs.W_STD, seed=100 + e, device=device)
        q = aq.aq_quantize(w, G, bits, scale_dtype=torch.bfloat16)
        wq[e].copy_(q[0]); sc[e].copy_(q[1]); bi[e].copy_(q[2])
    tok, offsets = inputs.moe_sort(inputs.moe_routing())
    x_tok = inputs.normal((inputs.MOE_TOKENS, K), 1.0, torch.bfloat16, seed=9, device=device)
    x_sorted = x_tok[tok.to(device)].contiguous()
    off_d = offsets.to(device)
    y = torch.empty(x_sorted.shape[0], N, dtype=torch.bfloat16, device=device)
    ms = time_calls(lambda: aq.aq_qmm_t_grouped(x_sorted, off_d, wq, sc, bi, G, bits, out=y), 10, stream)
    moe_bytes = E * N * (K * bits // 8 + 4 * (K // G)) + 2 * x_sorted.numel() + 2 * y.numel()
    hbm, _ = hbm_peak()
    out["moe_w8_g32"] = {"experts": E, "W": [N, K], "rows": int(x_sorted.shape[0]), "us": round(ms * 1e3, 2),
                         "GBps": round(moe_bytes / ms / 1e6, 1), "frac_of_hbm_peak": round(moe_bytes / ms / 1e6 / hbm, 4)}
    del wq, sc, bi, x_sorted, y
    return out


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, else nvidia-smi)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self.reasons = set()
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        while not self._stop.is_set():
            try:
                if self._nvml is not None:
                    p = self._nvml
                    self.samples.append(p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM))
                    try:
                        mask = p.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    except Exception:
                        mask = p.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                    for bit, name in self.REASONS.items():
                        if mask & bit:
                            self.reasons.add(name)
                else:
                    out = subprocess.run(
                        ["nvidia-smi", f"--id={self.index}", "--query-gpu=clocks.sm,clocks.max.sm,"
                         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                         "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5).stdout
                    f = [v.strip() for v in out.strip().split(",")]
                    self.samples.append(float(f[0]))
                    self.max_mhz = float(f[1])
                    for name, val in zip(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                          "sw_power_cap"], f[2:]):
                        if val.lower() == "active":
                            self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=10)

    def summary(self):
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(s)}


# ---------------------------------------------------------------------------
# peaks and committed ncu traffic
# ---------------------------------------------------------------------------

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources the warp-level kernel is compiled from (its translation units and every csrc header
# they include): its committed DRAM counters stay valid while these are unchanged
WARP_KERNEL_SOURCES = ("aq_internal.h", "device_common.cuh", "kernels_warp_mma.cu", "kernels_warp_mma_b2.cu",
                       "kernels_warp_mma_b4.cu", "kernels_warp_mma_b8.cu", "sm100_ptx.cuh", "warp_mma.cuh",
                       "warp_mma_kernel.cuh")


def committed_traffic(kernel_tag: str):
    """Per-launch DRAM bytes of `kernel_tag` from the committed ncu summary, if the
    kernel's sources have not changed since the capture (their hash is recorded there)."""
    import hashlib
    summ = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(summ):
        return None
    src_hash = hashlib.sha256()
    for name in WARP_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "group_wise_affine_qmv_b200", "csrc", name), "rb") as f:
            src_hash.update(f.read())
    cur = src_hash.hexdigest()[:16]
    for line in open(summ):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_tag and parts[1] == cur:
            try:
                return float(parts[2])
            except ValueError:
                return None
    return None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def build_workload(device, layers):
    """Distinct quantized weights for every matrix of the step (seeded, quantized on the device)
    and the activation buffers of the chain, per bit width."""
    from group_wise_affine_qmv_b200 import aq
    W = {}
    seed = 1000
    for bits in BITS_LIST:
        lay = []
        for layer in range(layers):
            mats = {}
            for name, K, N in inputs.DECODE_PROJ:
                seed += 1
                w = inputs.decode_w(K, N, seed, device=device)
                mats[name] = aq.aq_quantize(w, GROUP, bits, scale_dtype=torch.bfloat16)
                del w
            lay.append(mats)
        seed += 1
        w = inputs.decode_w(inputs.LM_HEAD[1], inputs.LM_HEAD[2], seed, device=device)
        W[bits] = {"layers": lay, "lm": aq.aq_quantize(w, GROUP, bits, scale_dtype=torch.bfloat16)}
        del w
    B = inputs.DECODE_BATCH
    mk = lambda n: torch.empty(B, 1, n, dtype=torch.bfloat16, device=device)
    A = {"h0": inputs.decode_x(HIDDEN, seed=7 + HIDDEN, device=device)}
    for bits in BITS_LIST:
        A[bits] = {"h": mk(HIDDEN), "q": mk(PROJ["q"][1]), "k": mk(PROJ["k"][1]), "v": mk(PROJ["v"][1]),
                   "a": mk(PROJ["gate"][1]), "logits": mk(inputs.LM_HEAD[2])}
    return W, A


def run_layers(W, A, bits):
    """The 28 chained decoder layers of one bit width (4 launches each): q, k, v from the
    RMS-normalised hidden state, o(v) added into it, gate/up + silu*mul from it normalised again,
    down added into it."""
    from group_wise_affine_qmv_b200 import aq
    Wb, Ab = W[bits], A[bits]
    h0, h = A["h0"], Ab["h"]
    for layer, m in enumerate(Wb["layers"]):
        x_in = h0 if layer == 0 else h
        aq.aq_qmm_t_multi(x_in, [m["q"], m["k"], m["v"]], GROUP, bits, outs=[Ab["q"], Ab["k"], Ab["v"]],
                          rms_eps=RMS_EPS)
        aq.aq_qmm_t_residual(Ab["v"], *m["o"], GROUP, bits, r=x_in, out=h)
        aq.aq_qmm_t_swiglu(h, m["gate"], m["up"], GROUP, bits, out=Ab["a"], rms_eps=RMS_EPS)
        aq.aq_qmm_t_residual(Ab["a"], *m["down"], GROUP, bits, r=h, out=h)
    return 4 * len(Wb["layers"])


def run_lm_head(W, A, bits):
    from group_wise_affine_qmv_b200 import aq
    aq.aq_qmm_t(A[bits]["h"], *W[bits]["lm"], GROUP, bits, out=A[bits]["logits"])
    return 1


def run_step(W, A):
    n = 0
    for bits in BITS_LIST:
        n += run_layers(W, A, bits)
        n += run_lm_head(W, A, bits)
    return n


def cpu_baseline(layers, budget_s=12.0):
    """The oracle as it stands, on a bounded row sample of the lm_head matrix (4-bit),
    scaled to GB/s of algorithmic bytes."""
    import numpy as np
    import oracle
    K, N = inputs.LM_HEAD[1], inputs.LM_HEAD[2]
    rows = 4096
    w = inputs.decode_w(K, rows, seed=424242)
    x = inputs.decode_x(K, seed=7 + K).reshape(inputs.DECODE_BATCH, K)
    Q = oracle.quantize(w.numpy(), GROUP, 4, "bf16")
    xb = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    done_rows = 0
    t0 = time.perf_counter()
    chunk = 256
    while time.perf_counter() - t0 < budget_s:
        lo = done_rows % rows
        codes = oracle.unpack(Q.packed[lo:lo + chunk], K, 4)
        wd = oracle.dequant(codes, Q.scale_bits[lo:lo + chunk], Q.bias_bits[lo:lo + chunk], GROUP, "bf16")
        oracle.linear_contig(xb, "bf16", wd)
        done_rows += chunk
    dt = time.perf_counter() - t0
    bytes_done = done_rows * (K * 4 // 8 + 2 * 2 * (K // GROUP)) + 2 * inputs.DECODE_BATCH * (K + done_rows)
    cores = len(os.sched_getaffinity(0))
    return {"value": bytes_done / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{done_rows} lm_head rows (K={K}, 4-bit, G={GROUP}) x 32 tokens: unpack + fp64 dequant "
                      f"+ fp64 contraction, {dt:.1f} s"}


def dist_setup(n_gpus):
    if n_gpus > 1 or "RANK" in os.environ:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, rank, world, local
    torch.cuda.set_device(0)
    return None, 0, 1, 0


def max_over_ranks(dist, value, device):
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        dist.barrier(device_ids=[device.index])
    torch.cuda.synchronize(device)


def device_error_on_any_rank(dist, stream, device):
    """Read and clear this rank's device error word; every rank learns whether any rank had one
    (so that all take the same next step).  Returns this rank's message, "another rank", or None."""
    from group_wise_affine_qmv_b200 import aq
    msg = None
    try:
        with torch.cuda.stream(stream):
            aq.aq_device_error()
    except aq.AQError as ex:
        msg = str(ex)
    if max_over_ranks(dist, 1.0 if msg else 0.0, device) > 0.0:
        return msg or "another rank"
    return None


def graph_of(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def time_graph(g, reps, stream, before=None):
    """Average device time (ms) of one replay of `g` (CUDA events on `stream`); `before`, when
    given, is replayed untimed ahead of every timed replay (to leave L2 as a step would)."""
    tot = 0.0
    with torch.cuda.stream(stream):
        g.replay()
        for _ in range(reps):
            if before is not None:
                before.replay()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            g.replay()
            a1.record(stream)
            a1.synchronize()
            tot += a0.elapsed_time(a1)
    return tot / reps


def unfused_sweep(W, A, bits, stream):
    """The same matrices as seven plain aq_qmm_t calls per layer, all on the fixed input h0
    (no call depends on another): the round-trip of the unfused step, for comparison."""
    from group_wise_affine_qmv_b200 import aq
    Ab = A[bits]
    outs = {"q": Ab["q"], "k": Ab["k"], "v": Ab["v"], "o": Ab["h"], "gate": Ab["a"], "up": Ab["a"]}
    a_in = Ab["a"]

    def sweep():
        for m in W[bits]["layers"]:
            for name, K, N in inputs.DECODE_PROJ:
                if name == "down":
                    aq.aq_qmm_t(a_in, *m[name], GROUP, bits, out=Ab["h"])
                else:
                    aq.aq_qmm_t(A["h0"], *m[name], GROUP, bits, out=outs[name])
    g = graph_of(sweep, stream)
    ms = time_graph(g, 10, stream)
    del g
    nbytes = sum(matrix_bytes(K, N, bits) for _, K, N in inputs.DECODE_PROJ) * len(W[bits]["layers"])
    return {"us": round(ms * 1e3, 1), "GBps": round(nbytes / ms / 1e6, 1), "launches": 7 * len(W[bits]["layers"])}


def ours(args):
    dist, rank, world, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    layers = args.layers
    W, A = build_workload(device, layers)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)
    nbytes = step_bytes(layers)

    # eager warm-up (also checks that every call succeeds), then capture one step
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            launches_per_step = run_step(W, A)
    torch.cuda.synchronize(device)
    graph = graph_of(lambda: run_step(W, A), stream)
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            graph.replay()
    torch.cuda.synchronize(device)

    # ---- device-resident timing.  A kernel that reports an expired bounded wait voids the run
    #      (its CTA gave up after 2 s): the timed loop is then measured once more, and the JSON
    #      line says so (`device_error_remeasured`); a second error ends the run. ----
    from group_wise_affine_qmv_b200 import aq
    remeasured = None
    for attempt in range(2):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dist, device)
        with ClockSampler(local) as clk:
            with torch.cuda.stream(stream):
                ev0.record(stream)
                for _ in range(args.steps):
                    graph.replay()
                ev1.record(stream)
            ev1.synchronize()
        err = device_error_on_any_rank(dist, stream, device)
        if err is None:
            break
        if attempt == 1:
            raise RuntimeError("timed loop measured twice, a kernel reported an error both times: " + err)
        remeasured = err
    barrier(dist, device)
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(dist, ms, device)
    ms_per_step = ms_max / args.steps
    value = world * nbytes * args.steps / (ms_max / 1e3) / 1e9

    # ---- per-bits breakdown: the 28 chained layers, lm_head alone after them (so that none of
    #      its weights are left in L2 from the previous call), and the unfused sweep ----
    detail = {}
    reps = max(20, args.steps // 10)
    hbm, _ = hbm_peak()
    layer_bytes = {}
    layer_ms = {}
    for bits in BITS_LIST:
        g_layers = graph_of(lambda: run_layers(W, A, bits), stream)
        glm = graph_of(lambda: run_lm_head(W, A, bits), stream)
        layers_ms = time_graph(g_layers, reps, stream)
        lm_ms = time_graph(glm, reps, stream, before=g_layers)
        K, N = inputs.LM_HEAD[1], inputs.LM_HEAD[2]
        lm_bytes = matrix_bytes(K, N, bits)
        lb = layers * sum(layer_launch_bytes(bits))
        layer_bytes[bits], layer_ms[bits] = lb, layers_ms
        per_launch = [round(v / 1e6, 3) for v in layer_launch_bytes(bits)]
        detail[f"w{bits}"] = {"layers_us": round(layers_ms * 1e3, 2), "layers_GBps": round(lb / layers_ms / 1e6, 1),
                              "layers_frac_of_peak": round(lb / layers_ms / 1e6 / hbm, 4),
                              "us_per_layer_launch": round(layers_ms * 1e3 / (4 * layers), 2),
                              "layer_launch_MB": per_launch,
                              "lm_head_us": round(lm_ms * 1e3, 2), "lm_head_GBps": round(lm_bytes / lm_ms / 1e6, 1),
                              "lm_head_frac_of_peak": round(lm_bytes / lm_ms / 1e6 / hbm, 4)}
        del g_layers, glm
        detail[f"w{bits}"]["unfused_sweep"] = unfused_sweep(W, A, bits, stream)

    # ---- end-to-end: input hidden state H2D, the step, logits D2H, per step.  The step runs as one
    #      graph per bit width; each width's logits go to pinned host memory on a copy stream as soon
    #      as its lm_head is done, overlapping the next part of the step, and a width's lm_head waits
    #      until the previous step's copy of its logits has been read out.  The timed region ends
    #      after the last copy. ----
    h_host = A["h0"].cpu().pin_memory()
    logits_host = {bits: torch.empty(A[bits]["logits"].shape, dtype=torch.bfloat16).pin_memory()
                   for bits in BITS_LIST}
    h2d = h_host.numel() * h_host.element_size()
    d2h = sum(t_.numel() * t_.element_size() for t_ in logits_host.values())
    e2e_steps = max(3, args.steps // 4)
    parts = {bits: graph_of(lambda b=bits: (run_layers(W, A, b), run_lm_head(W, A, b)), stream) for bits in BITS_LIST}
    copy_stream = torch.cuda.Stream(device)
    done = {bits: torch.cuda.Event() for bits in BITS_LIST}
    copied = {bits: torch.cuda.Event() for bits in BITS_LIST}
    e2e_error = None
    for attempt in range(2):   # measured once more if a kernel reported an expired wait
        torch.cuda.synchronize(device)
        barrier(dist, device)
        with torch.cuda.stream(stream):
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for step in range(e2e_steps):
                A["h0"].copy_(h_host, non_blocking=True)
                for bits in BITS_LIST:
                    if step > 0:
                        stream.wait_event(copied[bits])
                    parts[bits].replay()
                    done[bits].record(stream)
                    copy_stream.wait_event(done[bits])
                    with torch.cuda.stream(copy_stream):
                        logits_host[bits].copy_(A[bits]["logits"], non_blocking=True)
                    copied[bits].record(copy_stream)
            for bits in BITS_LIST:
                stream.wait_event(copied[bits])
            f1.record(stream)
        f1.synchronize()
        err = device_error_on_any_rank(dist, stream, device)
        if err is None:
            break
        if attempt == 1:
            raise RuntimeError("end-to-end loop measured twice, a kernel reported an error both times: " + err)
        e2e_error = err
    del parts
    barrier(dist, device)
    e2e_ms = max_over_ranks(dist, f0.elapsed_time(f1), device)
    e2e_value = world * nbytes * e2e_steps / (e2e_ms / 1e3) / 1e9

    # ---- roofline of the dominant kernel: the warp-level kernel runs every layer launch ----
    peak, peak_kind = hbm_peak()
    lb_all = sum(layer_bytes.values())
    lms_all = sum(layer_ms.values())
    n_layer_launches = 4 * layers * len(BITS_LIST)
    per_launch_bytes = lb_all / n_layer_launches
    per_launch_s = lms_all / 1e3 / n_layer_launches
    achieved = per_launch_bytes / per_launch_s / 1e9
    traffic = committed_traffic("qmm_warp_kernel_decode_chain")

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights quantized on the device, N(0,1) input hidden state)",
        "config": bench_config(layers, world),
        "detail": detail,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "qmm_warp_kernel (every layer launch of the step; lm_head in detail)",
                     "bytes_per_launch": round(per_launch_bytes), "peak_source": peak_kind},
        "clocks": clk.summary(),
    }
    if remeasured is not None:
        result["device_error_remeasured"] = remeasured
    if e2e_error is not None:
        result["e2e"]["device_error_remeasured"] = e2e_error
    if not args.no_prefill:
        result["detail"]["prefill"] = prefill_and_moe(device, stream)
        result["detail"]["probe_and_ragged_qmv"] = probe_and_ragged(device, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(layers)
    if rank == 0:
        print(json.dumps(result), flush=True)
    del graph
    if dist is not None:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on a bounded sample per step
# ---------------------------------------------------------------------------

def reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    layers = args.layers
    # per step: a bounded row sample of every matrix shape of the sweep, 4- and 8-bit
    shapes = sorted({(K, N) for _, K, N in sweep_shapes(layers)})
    rows_per_matrix = 8
    prepared = []
    for bits in BITS_LIST:
        for (K, N) in shapes:
            w = inputs.decode_w(K, rows_per_matrix, seed=K * 7 + N + bits)
            Q = oracle.quantize(w.numpy(), GROUP, bits, "bf16")
            x = inputs.decode_x(K, seed=7 + K).reshape(inputs.DECODE_BATCH, K)
            prepared.append((bits, K, Q, x.contiguous().view(torch.int16).numpy().view(np.uint16)))

    def step():
        b = 0
        for bits, K, Q, xb in prepared:
            codes = oracle.unpack(Q.packed, K, bits)
            wd = oracle.dequant(codes, Q.scale_bits, Q.bias_bits, GROUP, "bf16")
            oracle.linear_contig(xb, "bf16", wd)
            b += rows_per_matrix * (K * bits // 8 + 4 * (K // GROUP)) + 2 * inputs.DECODE_BATCH * (K + rows_per_matrix)
        return b

    for _ in range(max(args.warmup, 3)):
        step()
    t0 = time.perf_counter()
    tot = 0
    for _ in range(args.steps):
        tot += step()
    dt = time.perf_counter() - t0
    value = tot / dt / 1e9
    cores = len(os.sched_getaffinity(0))
    sample = (f"{rows_per_matrix} rows of each of the {len(shapes)} matrix shapes of the sweep, bits 4 and 8, "
              f"x 32 tokens per step")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(layers, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


CASES = ("lm_head_w4", "lm_head_w8", "lm_head2x_w4", "prefill_w4", "prefill_w8", "k_w4", "k_w8", "down_w4",
         "down_w8", "qkv_w4", "qkv_w8", "gateup_w4", "gateup_w8", "layer_w4", "layer_w8", "step")


def step_case(reps):
    """The timed decode step (28 layers and lm_head, bits 4 and 8: 226 launches), run eagerly once to
    warm up and then `reps` times, for a launch list of exactly one or more steps."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    W, A = build_workload(device, inputs.DECODE_LAYERS)
    run_step(W, A)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(reps):
        launches = run_step(W, A)
    a1.record(stream)
    a1.synchronize()
    from group_wise_affine_qmv_b200 import aq
    aq.aq_device_error()
    print(json.dumps({"case": "step", "launches_per_step": launches, "reps": reps,
                      "ms_per_step": round(a0.elapsed_time(a1) / reps, 4), "graph": False}), flush=True)


def single_case(name, reps):
    """One shape alone, for profiling: `reps` timed calls after two warm-up calls (CUDA events).
    lm_head*: x [32, 1, 1024] against W [151936, 1024] (2x: 303872 rows, > L2); k*, down*: x
    [32, 1, K] against the decode step's k (W [1024, 1024]) or down (W [1024, 3072]) projection;
    qkv*: the fused q/k/v call; gateup*: the fused gate/up + silu*mul call; layer*: the four
    chained launches of one decoder layer; prefill*: x [2, 2048, 4096] against W [14336, 4096];
    G = 64, weights quantized on the device."""
    from group_wise_affine_qmv_b200 import aq
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    bits = int(name[-1])
    B = inputs.DECODE_BATCH
    if name.startswith(("qkv", "gateup", "layer")):
        W, A = build_workload(device, 1)
        W = {bits: W[bits]}
        m = W[bits]["layers"][0]
        Ab = A[bits]
        if name.startswith("qkv"):
            fn = lambda: aq.aq_qmm_t_multi(A["h0"], [m["q"], m["k"], m["v"]], GROUP, bits,
                                           outs=[Ab["q"], Ab["k"], Ab["v"]], rms_eps=RMS_EPS)
            nbytes = layer_launch_bytes(bits)[0]
        elif name.startswith("gateup"):
            fn = lambda: aq.aq_qmm_t_swiglu(A["h0"], m["gate"], m["up"], GROUP, bits, out=Ab["a"], rms_eps=RMS_EPS)
            nbytes = layer_launch_bytes(bits)[2]
        else:
            fn = lambda: run_layers(W, A, bits)
            nbytes = sum(layer_launch_bytes(bits))
        ms = time_calls(fn, reps, torch.cuda.current_stream())
        aq.aq_device_error()
        print(json.dumps({"case": name, "bits": bits, "us": round(ms * 1e3, 2), "GBps": round(nbytes / ms / 1e6, 1)}),
              flush=True)
        return
    if name.startswith(("lm_head", "k_", "down_")):
        if name.startswith("lm_head"):
            K, N = 1024, inputs.LM_HEAD[2] * (2 if name.startswith("lm_head2x") else 1)
        else:
            _, K, N = {p[0]: p for p in inputs.DECODE_PROJ}[name.split("_")[0]]
        x = inputs.decode_x(K, device=device)
        y = torch.empty(B, 1, N, dtype=torch.bfloat16, device=device)
        M = B
    else:
        K, N = inputs.PREFILL_W_UP[1], inputs.PREFILL_W_UP[0]
        x = inputs.normal((2, 2048, K), 1.0, torch.bfloat16, seed=5, device=device)
        y = torch.empty(2, 2048, N, dtype=torch.bfloat16, device=device)
        M = 2 * 2048
    w = inputs.normal((N, K), inputs.W_STD, seed=6, device=device)
    wq, sc, bi = aq.aq_quantize(w, GROUP, bits, scale_dtype=torch.bfloat16)
    del w
    ms = time_calls(lambda: aq.aq_qmm_t(x, wq, sc, bi, GROUP, bits, out=y), reps, torch.cuda.current_stream())
    aq.aq_device_error()
    nbytes = matrix_bytes(K, N, bits, M)
    print(json.dumps({"case": name, "M": M, "N": N, "K": K, "bits": bits, "us": round(ms * 1e3, 2),
                      "GBps": round(nbytes / ms / 1e6, 1), "TFLOPs": round(2.0 * M * N * K / ms / 1e9, 1)}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=inputs.DECODE_LAYERS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill / expert-bank detail")
    ap.add_argument("--case", choices=CASES, help="time one shape alone (profiling) instead of the benchmark")
    ap.add_argument("--reps", type=int, default=3, help="timed calls of --case")
    args = ap.parse_args()
    if args.case == "step":
        step_case(args.reps)
        return
    if args.case:
        single_case(args.case, args.reps)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
