"""Benchmark of the INT4 linear-layer hot path on B200 (one JSON line on rank 0).

Headline workload: the LLaMA-3.2-1B-shaped decode step, W4A16 at m = 1 -- 16 layers x {q 2048x2048,
k 512x2048, v 512x2048, o 2048x2048, gate 8192x2048, up 8192x2048, down 2048x8192}, asymmetric
group-128 INT4 weights ~N(0, 0.02^2) with 0.1% outliers x20, bf16 activations ~N(0, 1), fp32
outputs.  One step = the 112 GEMVs in the dependency structure of a decoder layer: 64 dependent stages
(per layer [q, k, v], o, [gate, up], down), each waiting for the previous one's outputs: 64 launches
with programmatic dependent launch, replayed from a CUDA graph.  The line also reports the same stages
as ONE q4_linear_w4a16_chain launch ("chain") and the chain with each down projection gated from its
layer's gate/up outputs.
Metric: HBM GB/s = algorithmic bytes (packed weights + fp16 scales + fp16 zeros + bf16 x + fp32 y)
of the step / device time of the step.

At one GPU the line also carries "components", the other rows of the hot path on their workloads:
  prefill  W4A16 GEMM, m = 2048, the same 112 weight matrices issued as a decoder layer can issue them
           at m > 4 ([q,k,v] and [gate,up] each one GEMM over stacked weights: 64 GEMMs), x with 1%
           of channels x10 (TFLOP/s); also at m = 64 and m = 512;
  w4a8     per-token INT8 act-quant + W4A8 GEMM, m = 4096, the same shapes quantized symmetrically and
           stacked the same way, Student-t(3) activations (TOPS); also at m = 16 and m = 256;
  moe      the MoE layer: 4096 tokens, hidden 2048, 64 experts of intermediate 1024, top-8 (tokens/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-components]
    python bench.py --ncu-case {decode-chain,decode-layer,gemm,prefill-m64,moe,moe-a8,moe-classes}
                                               (small launch sequences for ncu captures)

Multi-GPU (torchrun): every rank runs an independent replica of the decode step (the step has no data
exchange); value = bytes of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_linear_layers_b200 import synth  # noqa: E402

METRIC = "INT4 GEMV HBM GB/s (M=1); W4A16/W4A8 GEMM TOPS; MoE layer tokens/s"
MOE = dict(T=4096, H=2048, I=1024, E=64, topk=8)


# ------------------------------------------------------------------------------------------------ #
# distributed plumbing
# ------------------------------------------------------------------------------------------------ #

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    """The largest value over all ranks (every rank takes part; NCCL on GPUs, gloo on CPU)."""
    if ws == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------ #
# clocks sampled during the timed region (NVML, every 10 ms)
# ------------------------------------------------------------------------------------------------ #

class ClockSampler:
    def __init__(self, device: int, period_s: float = 0.002):
        self.period, self.samples, self.reasons, self.handle, self.max_mhz = period_s, [], set(), None, None
        self.power = []
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.nv = nv
            self.handle = nv.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.error = repr(e)
            self.handle = None

    def _run(self):
        nv = self.nv
        names = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                 "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                 "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                 "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        while not self.stop:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
                self.power.append(nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        self.stop = False
        if self.handle is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *a):
        self.stop = True
        if self.handle is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "power_w_max": round(max(self.power), 1) if self.power else None}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained") or d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


_INT8_PEAK = {}


def measure_int8_peak(dev):
    """A library int8 matmul on this GPU, timed like the driver's bf16 peak: torch._int_mm (cuBLASLt) on
    8192^3 int8 -> int32, best of 10 (TOPS = 2 N^3 / time).  Cached for the run."""
    if "tops" in _INT8_PEAK:
        return _INT8_PEAK["tops"]
    n = 8192
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t().contiguous().t()
    best = None
    try:
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1)
            best = t if best is None else min(best, t)
        _INT8_PEAK["tops"] = 2 * n ** 3 / (best * 1e-3) / 1e12
    except RuntimeError as e:   # no int8 matmul in this torch build: fall back to the nominal ratio
        _INT8_PEAK["tops"] = None
        _INT8_PEAK["error"] = str(e)[:200]
    del a, b
    return _INT8_PEAK["tops"]


def tensor_peak(peaks, clocks, int8=False):
    """The tensor-core denominator for a GEMM timed in this run: the burst figure when the timed region
    ran at the maximum SM clock with no power capping, the sustained one otherwise.  int8: the measured
    int8 matmul peak (burst), scaled by bf16 sustained / burst for the sustained case; 2 x bf16 when no int8
    peak was measured (the nominal dense ratio)."""
    burst = bool(clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]
                 and "sw_power_cap" not in clocks.get("reasons", []))
    bf = peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]
    kind = "burst" if burst else "sustained"
    if not int8:
        return bf, f"{peaks['source']} cuBLAS bf16, {kind} (clocks {clocks.get('sm_mhz')} of {clocks.get('sm_max_mhz')} MHz)"
    i8 = _INT8_PEAK.get("tops")
    if i8:
        v = i8 if burst else i8 * peaks["bf16_tflops_sustained"] / peaks["bf16_tflops"]
        return v, f"int8 torch._int_mm 8192^3 measured in this run ({round(i8, 1)} TOPS burst), {kind}"
    return 2 * bf, f"{peaks['source']} bf16 {kind} x 2 (nominal int8:bf16 dense ratio; int8 not measured)"


def traffic_from_profiles(name):
    """DRAM bytes per launch from an ncu capture (profiles/traffic.txt: `name bytes sha256-of-source
    source-path`), or None when there is none or the kernel source has changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        lines = fh.readlines()
    for line in lines:
        f = line.split()
        if len(f) == 4 and f[0] == name:
            src = os.path.join(ROOT, f[3])
            if os.path.exists(src):
                with open(src, "rb") as fs:
                    if hashlib.sha256(fs.read()).hexdigest() == f[2]:
                        return int(float(f[1]))
    return None


def graph_of(fn):
    """Capture fn in a CUDA graph after one eager call.  The eager call must finish within seconds: a call
    that takes longer ran into a kernel's bounded wait (10 s, Q4_ERR_TIMEOUT), and timing it would only
    measure the limit, so the run stops there."""
    t0 = time.time()
    fn()
    torch.cuda.synchronize()
    if time.time() - t0 > 5.0:
        raise SystemExit(f"bench: an eager call took {time.time() - t0:.1f} s (a bounded wait ran out?); not timing it")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_replays(g, steps, ws, sampler=None):
    stream = torch.cuda.current_stream()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (sampler if sampler is not None else _Null()):
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if sampler is not None and sampler.handle is not None:
            # a short timed region yields one or two clock readings: keep the same load running (untimed,
            # after e1) until the sampler holds 20 readings of it or half a second has passed
            t_end = time.time() + 0.5
            while len(sampler.samples) < 20 and time.time() < t_end:
                g.replay()
                torch.cuda.synchronize()
    barrier(ws)
    return max_over_ranks(e0.elapsed_time(e1), ws)


def dev_bf16(a_u16, dev):
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).to(dev).view(torch.bfloat16)


# ------------------------------------------------------------------------------------------------ #
# workloads
# ------------------------------------------------------------------------------------------------ #

def decode_layers(n_layers=synth.LLAMA_1B_LAYERS):
    return [(f"L{l}.{nm}", n, k) for l in range(n_layers) for (nm, n, k) in synth.LLAMA_1B_LINEARS]


def decode_bytes(layers):
    """Algorithmic HBM bytes of one decode step: packed weights, fp16 scales and zeros, bf16 x, fp32 y."""
    return sum(n * k // 2 + 2 * 2 * n * (k // 128) + 2 * k + 4 * n for (_, n, k) in layers)


def footprint(layers):
    """Bytes of the step's linears as INT4 (packed codes + fp16 scales (+ fp16 zeros), group 128) against
    fp16 weights: the INT4+MoE page's "about 1/4 of FP16 memory"."""
    fp16 = sum(2 * n * k for (_, n, k) in layers)
    asym = sum(n * k // 2 + 2 * 2 * n * (k // 128) for (_, n, k) in layers)
    sym = sum(n * k // 2 + 2 * n * (k // 128) for (_, n, k) in layers)
    return {"fp16_bytes": fp16, "int4_asym_g128_bytes": asym, "int4_sym_g128_bytes": sym,
            "ratio_asym_g128": round(asym / fp16, 4), "ratio_sym_g128": round(sym / fp16, 4),
            "pages": "about 1/4 (INT4+MoE page, the effect of INT4 quantization on LLaMA 3.2-1B)"}


def build_weights(q4, dev, symmetric_too: bool, seed=0):
    """The 112 weight matrices quantized on the device (asymmetric, and symmetric when asked)."""
    asym, sym = [], []
    for (name, n, k) in decode_layers():
        W = torch.from_numpy(synth.weights((seed, "llama1b", name), n, k)).to(dev)
        asym.append(q4.q4_quantize_pack(W, 128, False))
        if symmetric_too:
            sym.append(q4.q4_quantize_pack(W, 128, True))
        del W
    torch.cuda.synchronize()
    return asym, sym


def run_decode(q4, args, ws, weights, dev):
    layers = decode_layers()
    # every linear has its own x and y; they live in two contiguous buffers (one host copy each way per
    # step for the end-to-end number), each slice 16-byte aligned
    x_all = dev_bf16(np.concatenate([synth.activations((0, "llama1b-decode-x", name), 1, k).reshape(-1)
                                     for (name, n, k) in layers]), dev)
    y_all = torch.empty(sum(n for (_, n, _) in layers), dtype=torch.float32, device=dev)
    xs, ys, ox, oy = [], [], 0, 0
    for (_, n, k) in layers:
        xs.append(x_all[ox:ox + k].view(1, k))
        ys.append(y_all[oy:oy + n].view(1, n))
        ox += k
        oy += n
    bytes_step = decode_bytes(layers)

    # per layer: [q, k, v] grouped, o, [gate, up] grouped, down (the dependency structure of a layer): 64
    # dependent stages per step
    stage_idx = []
    for l in range(synth.LLAMA_1B_LAYERS):
        b = 7 * l
        stage_idx += [(b, b + 1, b + 2), (b + 3,), (b + 4, b + 5), (b + 6,)]
    # the headline: one launch per stage (q4_linear_w4a16_grouped for [q,k,v] and [gate,up], one problem
    # for o and down; programmatic dependent launch lets a stage's CTAs stream their weights while the
    # previous stage runs): 64 launches per step
    calls = [q4.GroupedGemv([xs[i] for i in idx], [weights[i] for i in idx], [ys[i] for i in idx]) for idx in stage_idx]

    def step():
        for c in calls:
            c()

    # the same step as ONE launch of the GEMV chain (stage s waits inside the kernel for stage s-1's outputs)
    chain = q4.GemvChain([[(xs[i].view(-1), weights[i], ys[i].view(-1)) for i in idx] for idx in stage_idx])

    def step_chain():
        chain()

    # the same step with the dense FFN chained: down consumes silu(gate) * up of this layer's [gate, up]
    # outputs inside the chain (a real data dependency)
    fused_stages = []
    for l in range(synth.LLAMA_1B_LAYERS):
        b = 7 * l
        fused_stages += [[(xs[i].view(-1), weights[i], ys[i].view(-1)) for i in (b, b + 1, b + 2)],
                         [(xs[b + 3].view(-1), weights[b + 3], ys[b + 3].view(-1))],
                         [(xs[i].view(-1), weights[i], ys[i].view(-1)) for i in (b + 4, b + 5)],
                         [((ys[b + 4].view(-1), ys[b + 5].view(-1)), weights[b + 6], ys[b + 6].view(-1))]]
    chain_fused = q4.GemvChain(fused_stages)
    bytes_fused = bytes_step + synth.LLAMA_1B_LAYERS * (2 * 4 * 8192 - 2 * 8192)   # down reads fp32 g, u

    g = graph_of(step)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    clk = ClockSampler(torch.cuda.current_device())
    ms = time_replays(g, args.steps, ws, clk)
    ms_step = ms / args.steps
    value = ws * bytes_step * args.steps / (ms * 1e-3) / 1e9

    gc = graph_of(step_chain)
    for _ in range(args.warmup):
        gc.replay()
    ms_c = time_replays(gc, args.steps, ws) / args.steps
    gf = graph_of(lambda: chain_fused())
    for _ in range(args.warmup):
        gf.replay()
    ms_f = time_replays(gf, args.steps, ws) / args.steps

    # end to end through the public calls with host buffers: the step's x (pinned host memory) copied in,
    # the 64 prepared calls issued eagerly, every y copied back to pinned host memory
    hx = x_all.cpu().pin_memory()
    hy = torch.empty(y_all.shape, dtype=y_all.dtype).pin_memory()
    h2d = hx.numel() * hx.element_size()
    d2h = hy.numel() * hy.element_size()

    def e2e_step():
        x_all.copy_(hx, non_blocking=True)
        for c in calls:
            c()
        hy.copy_(y_all, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    stream = torch.cuda.current_stream()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(f0.elapsed_time(f1), ws)
    e2e_val = ws * bytes_step * args.steps / (ms_e2e * 1e-3) / 1e9

    peaks = load_peaks()
    per_gpu = value / ws
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "llama-3.2-1b-shaped decode step: W4A16 GEMV m=1 over 16 layers x 7 linears "
                               "(q,k,v,o 2048/512/512/2048 x 2048, gate/up 8192x2048, down 2048x8192), "
                               "asymmetric INT4 group 128, bf16 x ~N(0,1), fp32 y",
                   "linears_per_step": len(layers), "bytes_per_step": bytes_step,
                   "memory_footprint": footprint(layers),
                   "l2": "no flush: the step streams %.0f MB of weights, > 126 MB L2" % (bytes_step / 1e6),
                   "launch": "64 dependent launches per step (per layer [q,k,v] and [gate,up] as "
                             "q4_linear_w4a16_grouped, o and down alone; programmatic dependent launch), replayed "
                             "from a CUDA graph",
                   "chain": {"ms_per_step": round(ms_c, 5), "value": round(bytes_step / (ms_c * 1e-3) / 1e9, 2),
                             "launch": "the same 64 stages as ONE q4_linear_w4a16_chain launch (each stage waits "
                                       "inside the kernel for the previous one's arrival counter)"},
                   "fused_swiglu_ffn": {"ms_per_step": round(ms_f, 5),
                                        "value": round(bytes_fused / (ms_f * 1e-3) / 1e9, 2),
                                        "launch": "the chain with down's input = silu(gate) * up of this layer's "
                                                  "[gate,up] outputs, read inside the same launch (a real dependency)"},
                   "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "hbm", "achieved": round(per_gpu, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(per_gpu / peaks["hbm_gbs"], 4), "traffic": traffic_from_profiles("gemv_decode"),
                     "peak_source": peaks["source"] + " (HBM copy bandwidth)",
                     "kernel": "w4a16_gemv_kernel; achieved = algorithmic bytes of the step / step time = bytes per "
                               "launch / mean launch duration (graph replay, gaps included)",
                     "mean_launch_us": round(1e3 * ms_step / len(calls), 3)},
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "eager public-API calls (64 prepared q4.GroupedGemv calls per step); all x of the step copied "
                       "in from pinned host memory and all y copied back to pinned host memory every step"},
        "gpu_launches": len(calls) * args.steps,
        "clocks": clk.summary(),
    }


def layer_gemms(q4, weights):
    """The 112 matrices issued the way a decoder layer can issue them at m > 4: [q,k,v] and [gate,up] (which
    read the same input) each as ONE GEMM over their stacked weights (Q4Weight.stack: the parts' quantized
    rows one after another, so the products are exactly the parts'), o and down alone: 64 GEMMs per step."""
    out = []
    for l in range(synth.LLAMA_1B_LAYERS):
        w = weights[7 * l: 7 * l + 7]
        out += [q4.Q4Weight.stack(w[0:3]), w[3], q4.Q4Weight.stack(w[4:6]), w[6]]
    return out


def gemm_launches(q4, gemms, m):
    """Kernel launches of one step: one per GEMM, plus the reduction of those split along K."""
    return sum(1 + (q4._lib.q4_linear_workspace_size(m, ctypes.byref(w.desc)) > 0) for w in gemms)


def run_prefill(q4, args, weights, dev, m=2048):
    layers = decode_layers()
    gemms = layer_gemms(q4, weights)
    xk = {k: dev_bf16(synth.activations((0, "llama1b-prefill-x", k), m, k, "outlier_channels"), dev)
          for k in sorted({k for (_, _, k) in layers})}
    yn = {w.n: torch.empty((m, w.n), dtype=torch.bfloat16, device=dev) for w in gemms}

    def step():
        for w in gemms:
            q4.q4_linear_w4a16(xk[w.k], w, y=yn[w.n])

    g = graph_of(step)
    for _ in range(3):
        g.replay()
    steps = max(3, min(args.steps, 10))
    clk = ClockSampler(torch.cuda.current_device())
    ms = time_replays(g, steps, 1, clk) / steps
    flops = 2 * m * sum(n * k for (_, n, k) in layers)
    tf = flops / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    cl = clk.summary()
    pk, src = tensor_peak(peaks, cl)
    return {"value": round(tf, 1), "unit": "TFLOP/s", "ms_per_step": round(ms, 3), "m": m,
            "workload": f"W4A16 GEMM over the 112 decode-step matrices at m={m} ([q,k,v] and [gate,up] each one "
                        "GEMM over stacked weights: 64 GEMMs), x with 1% channels x10, bf16 out",
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk, "unit": "TFLOP/s",
                         "frac": round(tf / pk, 4), "frac_of_burst_peak": round(tf / peaks["bf16_tflops"], 4),
                         "peak_source": src},
            "gpu_launches": gemm_launches(q4, gemms, m) * steps, "clocks": cl}


def run_w4a8(q4, args, weights_sym, dev, m=4096):
    layers = decode_layers()
    xk = {k: dev_bf16(synth.activations((0, "llama1b-w4a8-x", k), m, k, "student_t3"), dev)
          for k in sorted({k for (_, _, k) in layers})}
    gemms = layer_gemms(q4, weights_sym)
    xq = {k: torch.empty((m, k), dtype=torch.int8, device=dev) for k in xk}
    sa = torch.empty((m,), dtype=torch.float32, device=dev)
    yn = {w.n: torch.empty((m, w.n), dtype=torch.bfloat16, device=dev) for w in gemms}

    def step():
        for w in gemms:   # one quantization of the GEMM's input, then the GEMM
            q4.act_quant_per_token(xk[w.k], xq=xq[w.k], scale_a=sa)
            q4.q4_linear_w4a8(xq[w.k], sa, w, y=yn[w.n])

    g = graph_of(step)
    for _ in range(3):
        g.replay()
    steps = max(3, min(args.steps, 10))
    clk = ClockSampler(torch.cuda.current_device())
    ms = time_replays(g, steps, 1, clk) / steps
    ops = 2 * m * sum(n * k for (_, n, k) in layers)
    tops = ops / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    cl = clk.summary()
    int8_peak, src = tensor_peak(peaks, cl, int8=True)
    return {"value": round(tops, 1), "unit": "TOPS", "ms_per_step": round(ms, 3), "m": m,
            "workload": "per-token INT8 act-quant + W4A8 GEMM over the 112 matrices (symmetric INT4 g128; [q,k,v] "
                        f"and [gate,up] each one GEMM over stacked weights: 64 GEMMs), m={m}, Student-t(3) "
                        "activations, bf16 out; act-quant time included",
            "roofline": {"bound": "tensor", "achieved": round(tops, 1), "peak": round(int8_peak, 1), "unit": "TOPS",
                         "frac": round(tops / int8_peak, 4), "peak_source": src},
            "gpu_launches": (gemm_launches(q4, gemms, m) + len(gemms)) * steps, "clocks": cl}


def with_attainable(r, m, a8: bool):
    """Adds the bound that the step's bytes put on a small-m GEMM: attainable = min(tensor peak, HBM
    bandwidth x arithmetic intensity), bytes = packed weights + scales (+ zeros) + activations in + bf16
    out, over the 112 matrices."""
    layers = decode_layers()
    peaks = load_peaks()
    g = 128
    wbytes = sum(n * k // 2 + n * (k // g) * 2 * (1 if a8 else 2) for (_, n, k) in layers)
    abytes = sum(m * k * (1 if a8 else 2) + (4 * m if a8 else 0) + 2 * m * n for (_, n, k) in layers)
    ops = 2 * m * sum(n * k for (_, n, k) in layers)
    inten = ops / (wbytes + abytes)
    peak = r["roofline"]["peak"]
    attain = min(peak, peaks["hbm_gbs"] * inten / 1e3)
    r["roofline"].update({"bytes_per_step": wbytes + abytes, "intensity_ops_per_byte": round(inten, 1),
                          "attainable": round(attain, 1), "frac_of_attainable": round(r["value"] / attain, 4),
                          "bound_at_this_m": "hbm" if attain < peak else "tensor"})
    return r


def build_moe(q4, dev, seed=0):
    T, H, I, E, topk = (MOE[k] for k in ("T", "H", "I", "E", "topk"))
    ex = []
    for nm, n, k in (("gate", E * I, H), ("up", E * I, H), ("down", E * H, I)):
        W = torch.from_numpy(synth.weights((seed, "moe", nm), n, k)).to(dev)
        ex.append(q4.q4_quantize_pack(W, 128, False))
        del W
    x = dev_bf16(synth.activations((seed, "moe", "x"), T, H), dev)
    Wr, bias = synth.router((seed, "moe"), E, H)
    return x, torch.from_numpy(Wr).to(dev), torch.from_numpy(bias).to(dev), tuple(ex)


MOE_TIERS = ((0, 3, 32), (3, 32, 64), (32, 64, 128))   # (first expert, end, group): hot, ordinary, cold


def tiered_classes(q4, dev):
    """The MoE workload's expert weights (the same fp32 matrices build_moe quantizes) cut into the hotness
    tiers, each quantized with its own group size (asymmetric)."""
    T, H, I, E, topk = (MOE[k] for k in ("T", "H", "I", "E", "topk"))
    cls = [[] for _ in MOE_TIERS]
    for nm, n_per, k in (("gate", I, H), ("up", I, H), ("down", H, I)):
        W = torch.from_numpy(synth.weights((0, "moe", nm), E * n_per, k)).to(dev)
        for c, (e0, e1, group) in enumerate(MOE_TIERS):
            cls[c].append(q4.q4_quantize_pack(W[e0 * n_per:e1 * n_per].contiguous(), group, False))
        del W
    return [t[0] for t in MOE_TIERS] + [E], [tuple(c) for c in cls]


def run_moe(q4, args, dev):
    T, H, I, E, topk = (MOE[k] for k in ("T", "H", "I", "E", "topk"))
    x, Wr, bias, ex = build_moe(q4, dev)
    ws_t = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk), dtype=torch.uint8, device=dev)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)

    g = graph_of(lambda: q4.moe_q4_forward(x, Wr, bias, topk, ex, I, y=y, workspace=ws_t))
    for _ in range(3):
        g.replay()
    steps = max(3, min(args.steps, 20))
    clk = ClockSampler(torch.cuda.current_device())
    ms = time_replays(g, steps, 1, clk) / steps
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    _, ids, _, _, _, counts = q4.moe_q4_forward(x, Wr, bias, topk, ex, I, workspace=ws_t, want_routing=True,
                                                dev_status=st)
    if int(st.item()) != 0:
        raise SystemExit(f"bench: the MoE layer reported device status {int(st.item())}")
    c = counts.cpu().numpy()
    flops = 2 * T * topk * 3 * H * I
    tf = flops / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    cl = clk.summary()
    pk, src = tensor_peak(peaks, cl)

    # the same layer with one shared expert of intermediate I (every token, weight 1)
    sh = []
    for nm, n, k in (("shared-gate", I, H), ("shared-up", I, H), ("shared-down", H, I)):
        W = torch.from_numpy(synth.weights((0, "moe", nm), n, k)).to(dev)
        sh.append(q4.q4_quantize_pack(W, 128, False))
        del W
    sh = tuple(sh)
    ws_s = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk, I), dtype=torch.uint8, device=dev)
    gs = graph_of(lambda: q4.moe_q4_forward(x, Wr, bias, topk, ex, I, y=y, workspace=ws_s, shared=sh))
    for _ in range(3):
        gs.replay()
    ms_s = time_replays(gs, steps, 1) / steps
    flops_s = flops + 2 * T * 3 * H * I
    # the same layer with the expert projections on per-row INT8 activation codes (moe_q4_forward_a8):
    # all three projections, and the down projection alone
    a8 = {}
    for name, mask in (("w4a8_experts", 3), ("w4a8_down_only", 2)):
        ws_a = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk, a8_mask=mask), dtype=torch.uint8, device=dev)
        ga = graph_of(lambda: q4.moe_q4_forward(x, Wr, bias, topk, ex, I, y=y, workspace=ws_a, a8_mask=mask))
        for _ in range(3):
            ga.replay()
        ms_a = time_replays(ga, steps, 1) / steps
        a8[name] = {"ms_per_step": round(ms_a, 4), "tokens_per_s": round(T / (ms_a * 1e-3), 1),
                    "tops": round(flops / (ms_a * 1e-3) / 1e12, 1), "a8_mask": mask}
        del ga, ws_a
    # the same layer with group sizes by expert hotness, the pages' three tiers: the 3 most chosen experts
    # (5 %; expert 0 is the hottest under the skew) at group 32, experts 3-31 at 64, 32-63 at 128
    begin, cls = tiered_classes(q4, dev)
    gc = graph_of(lambda: q4.moe_q4_forward_classes(x, Wr, bias, topk, begin, cls, I, y=y, workspace=ws_t))
    for _ in range(3):
        gc.replay()
    ms_c = time_replays(gc, steps, 1) / steps
    del gc
    return {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "workload": "MoE layer: 4096 tokens, hidden 2048, 64 SwiGLU experts of intermediate 1024, top-8, "
                        "asymmetric INT4 g128, fp32 router with Zipf-skewed logits (bias -1.1 ln(e+1)), fp32 out",
            "tflops": round(tf, 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk, "unit": "TFLOP/s",
                         "frac": round(tf / pk, 4), "frac_of_burst_peak": round(tf / peaks["bf16_tflops"], 4),
                         "peak_source": src, "algorithmic_flop": flops},
            "expert_counts": {"max": int(c.max()), "mean": float(c.mean()), "min": int(c.min()),
                              "empty": int((c == 0).sum())},
            "with_shared_expert": {"ms_per_step": round(ms_s, 4), "tokens_per_s": round(T / (ms_s * 1e-3), 1),
                                   "tflops": round(flops_s / (ms_s * 1e-3) / 1e12, 1),
                                   "workload": "the same layer plus one shared SwiGLU expert of intermediate "
                                               "1024 (moe_q4_forward_ex)"},
            "w4a8_experts": dict(a8["w4a8_experts"], workload="the same layer, gate/up and down on per-row INT8 "
                                 "activation codes, INT32 group partials (moe_q4_forward_a8, mask 3)"),
            "w4a8_down_only": dict(a8["w4a8_down_only"], workload="the same layer, only the down projection on "
                                   "INT8 codes of h (moe_q4_forward_a8, mask 2)"),
            "group_by_hotness": {"ms_per_step": round(ms_c, 4), "tokens_per_s": round(T / (ms_c * 1e-3), 1),
                                 "tflops": round(flops / (ms_c * 1e-3) / 1e12, 1),
                                 "workload": "the same layer with group sizes by expert hotness: experts 0-2 at "
                                             "group 32, 3-31 at 64, 32-63 at 128 (moe_q4_forward_classes)"},
            "gpu_launches": 6 * steps, "clocks": clk.summary()}


# ------------------------------------------------------------------------------------------------ #
# CPU baseline: the oracle on a bounded sample of the workload
# ------------------------------------------------------------------------------------------------ #

def oracle_decode_sample(rows_per_linear=128):
    """The oracle over the first rows of layer 0's seven linears (same weights and x as the device run).
    Returns (bytes processed, seconds)."""
    import oracle
    jobs = []
    for (name, n, k) in decode_layers(1):
        W = synth.weights((0, "llama1b", name), n, k)[:rows_per_linear]
        x = synth.activations((0, "llama1b-decode-x", name), 1, k)
        pk, sc, zr = oracle.quantize(W, 128, False)
        jobs.append((x, pk, sc, zr, rows_per_linear, k))
    t0 = time.perf_counter()
    for (x, pk, sc, zr, n, k) in jobs:
        oracle.linear_w4a16(x, pk, sc, zr, n, k, 128, False)
    dt = time.perf_counter() - t0
    nbytes = sum(n * k // 2 + 4 * n * (k // 128) + 2 * k + 4 * n for (_, _, _, _, n, k) in jobs)
    return nbytes, dt


def oracle_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline_decode(budget_s=10.0):
    b, t = oracle_decode_sample()
    reps = int(min(200, max(1, budget_s / max(t, 1e-3))))
    tb, tt = 0, 0.0
    for _ in range(reps):
        b, t = oracle_decode_sample()
        tb += b
        tt += t
    return {"value": round(tb / tt / 1e9, 4), "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{reps} passes of the oracle (fp64, OpenMP over output rows) over the first 128 rows of "
                      "layer 0's 7 linears, W4A16 m=1"}


def run_reference(args, ws, rank):
    """--impl reference: the oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_decode_sample()
    tb, tt = 0, 0.0
    for _ in range(args.steps):
        b, t = oracle_decode_sample()
        tb += b
        tt += t
    v = tb / tt / 1e9
    sample = "first 128 rows of layer 0's 7 linears per step (W4A16 m=1, fp64)"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tt / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "llama-3.2-1b-shaped decode step, W4A16 GEMV m=1 (oracle on a sample: "
                                   + sample + ")", "parallelism": "host cores"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def ncu_case(case):
    """Small, fixed launch sequences for ncu captures (each runs twice and exits; nothing is timed)."""
    from moe_linear_layers_b200 import q4
    dev = torch.device("cuda", torch.cuda.current_device())
    if case == "decode-chain":
        # the chain over six distinct layers (24 stages, 195 MB of weights > L2), launched twice
        layers = decode_layers(6)
        ws = []
        for (name, n, k) in layers:
            ws.append(q4.q4_quantize_pack(torch.from_numpy(synth.weights((0, "llama1b", name), n, k)).to(dev), 128, False))
        xs = [dev_bf16(synth.activations((0, "llama1b-decode-x", name), 1, k), dev).view(-1) for (name, n, k) in layers]
        ys = [torch.empty((n,), dtype=torch.float32, device=dev) for (_, n, _) in layers]
        stages = []
        for l in range(6):
            b = 7 * l
            stages += [[(xs[i], ws[i], ys[i]) for i in idx] for idx in ((b, b + 1, b + 2), (b + 3,), (b + 4, b + 5), (b + 6,))]
        chain = q4.GemvChain(stages)
        torch.cuda.synchronize()
        for _ in range(2):
            chain()
    elif case == "decode-layer":
        # six distinct layers (195 MB of weights > L2): [q,k,v] grouped, o, [gate,up] grouped, down
        layers = decode_layers(6)
        ws = []
        for (name, n, k) in layers:
            ws.append(q4.q4_quantize_pack(torch.from_numpy(synth.weights((0, "llama1b", name), n, k)).to(dev), 128, False))
        xs = [dev_bf16(synth.activations((0, "llama1b-decode-x", name), 1, k), dev) for (name, n, k) in layers]
        ys = [torch.empty((1, n), dtype=torch.float32, device=dev) for (_, n, _) in layers]
        torch.cuda.synchronize()
        for _ in range(2):
            for l in range(6):
                b = 7 * l
                q4.q4_linear_w4a16_grouped(xs[b:b + 3], ws[b:b + 3], ys[b:b + 3])
                q4.q4_linear_w4a16(xs[b + 3], ws[b + 3], y=ys[b + 3])
                q4.q4_linear_w4a16_grouped(xs[b + 4:b + 6], ws[b + 4:b + 6], ys[b + 4:b + 6])
                q4.q4_linear_w4a16(xs[b + 6], ws[b + 6], y=ys[b + 6])
    elif case == "gemm":
        # W4A16 m=2048 gate-shaped (8192x2048), then act-quant + W4A8 m=4096 of the same shape
        W = torch.from_numpy(synth.weights((0, "llama1b", "L0.gate"), 8192, 2048)).to(dev)
        wa, ws_ = q4.q4_quantize_pack(W, 128, False), q4.q4_quantize_pack(W, 128, True)
        x = dev_bf16(synth.activations((0, "llama1b-prefill-x", 2048), 2048, 2048, "outlier_channels"), dev)
        x8 = dev_bf16(synth.activations((0, "llama1b-w4a8-x", 2048), 4096, 2048, "student_t3"), dev)
        y = torch.empty((2048, 8192), dtype=torch.bfloat16, device=dev)
        y8 = torch.empty((4096, 8192), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        for _ in range(2):
            q4.q4_linear_w4a16(x, wa, y=y)
        for _ in range(2):
            xq, sa = q4.act_quant_per_token(x8)
            q4.q4_linear_w4a8(xq, sa, ws_, y=y8)
    elif case == "prefill-m64":
        # one decoder layer's seven W4A16 GEMMs at m = 64 (split along K), twice
        layers = decode_layers(1)
        ws = [q4.q4_quantize_pack(torch.from_numpy(synth.weights((0, "llama1b", name), n, k)).to(dev), 128, False)
              for (name, n, k) in layers]
        xs = {k: dev_bf16(synth.activations((0, "llama1b-prefill-x", k), 64, k, "outlier_channels"), dev)
              for (_, _, k) in layers}
        ys = [torch.empty((64, n), dtype=torch.bfloat16, device=dev) for (_, n, _) in layers]
        torch.cuda.synchronize()
        for _ in range(2):
            for w, (_, n, k), y in zip(ws, layers, ys):
                q4.q4_linear_w4a16(xs[k], w, y=y)
    elif case == "moe":
        T, H, I, E, topk = (MOE[k] for k in ("T", "H", "I", "E", "topk"))
        x, Wr, bias, ex = build_moe(q4, dev)
        ws_t = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk), dtype=torch.uint8, device=dev)
        y = torch.empty((T, H), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        for _ in range(2):
            q4.moe_q4_forward(x, Wr, bias, topk, ex, I, y=y, workspace=ws_t)
    elif case == "moe-classes":
        T, H, I, E, topk = (MOE[k] for k in ("T", "H", "I", "E", "topk"))
        x, Wr, bias, _ = build_moe(q4, dev)
        begin, cls = tiered_classes(q4, dev)
        ws_t = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk), dtype=torch.uint8, device=dev)
        y = torch.empty((T, H), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        for _ in range(2):
            q4.moe_q4_forward_classes(x, Wr, bias, topk, begin, cls, I, y=y, workspace=ws_t)
    elif case == "moe-a8":
        T, H, I, E, topk = (MOE[k] for k in ("T", "H", "I", "E", "topk"))
        x, Wr, bias, ex = build_moe(q4, dev)
        ws_t = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk, a8_mask=3), dtype=torch.uint8, device=dev)
        y = torch.empty((T, H), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        for _ in range(2):
            q4.moe_q4_forward(x, Wr, bias, topk, ex, I, y=y, workspace=ws_t, a8_mask=3)
    torch.cuda.synchronize()
    print(f"ncu case {case}: done", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", choices=["decode-chain", "decode-layer", "gemm", "prefill-m64", "moe", "moe-a8",
                                           "moe-classes"],
                    help="run a small fixed launch sequence for an ncu capture and exit (no JSON line)")
    args = ap.parse_args()
    if args.ncu_case:
        ncu_case(args.ncu_case)
        return

    if args.impl == "reference":
        line = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    args.warmup = max(args.warmup, 3)
    ws, rank, local = dist_setup()
    from moe_linear_layers_b200 import q4
    dev = torch.device("cuda", torch.cuda.current_device())
    components = ws == 1 and not args.no_components
    if components:
        measure_int8_peak(dev)
    asym, sym = build_weights(q4, dev, symmetric_too=components)
    line = run_decode(q4, args, ws, asym, dev)
    if components:
        line["components"] = {"prefill_w4a16_m2048": run_prefill(q4, args, asym, dev),
                              "w4a8_m4096": run_w4a8(q4, args, sym, dev)}
        # the other token counts of the prefill and W4A8 workloads, each against the bound its bytes set
        for m in (64, 512):
            line["components"][f"prefill_w4a16_m{m}"] = with_attainable(run_prefill(q4, args, asym, dev, m=m), m, False)
        for m in (16, 256):
            line["components"][f"w4a8_m{m}"] = with_attainable(run_w4a8(q4, args, sym, dev, m=m), m, True)
        del sym
        torch.cuda.empty_cache()
        line["components"]["moe_layer"] = run_moe(q4, args, dev)
        line["components"]["int8_peak_tops"] = {"value": _INT8_PEAK.get("tops") and round(_INT8_PEAK["tops"], 1),
                                                "how": "torch._int_mm int8 8192^3 -> int32, best of 10",
                                                **({"error": _INT8_PEAK["error"]} if "error" in _INT8_PEAK else {})}
    if rank == 0:
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_decode()
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
