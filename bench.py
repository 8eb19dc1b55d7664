"""Benchmark of the INT4 linear-layer hot path on B200.

Default workload (one JSON line): the LLaMA-3.2-1B-shaped decode step, W4A16 at m = 1: 16 layers x
{q 2048x2048, k 512x2048, v 512x2048, o 2048x2048, gate 8192x2048, up 8192x2048, down 2048x8192},
asymmetric group-128 INT4, bf16 activations ~N(0,1), fp32 outputs.  One step = the 112 GEMVs.
Metric: HBM GB/s = algorithmic bytes (packed weights + scales + zeros + x + y) / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Multi-GPU (torchrun, one rank per GPU): every rank runs an independent replica of the step (the
decode step has no data exchange); value = bytes of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_linear_layers_b200 import synth  # noqa: E402

METRIC = "INT4 GEMV HBM GB/s (M=1); W4A16/W4A8 GEMM TOPS; MoE layer tokens/s"


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
    if ws == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------ #
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------------ #

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        # nvidia-smi numbers GPUs differently from CUDA under CUDA_VISIBLE_DEVICES: select by UUID
        try:
            u = str(torch.cuda.get_device_properties(device).uuid)
            self.index = u if u.startswith("GPU-") else f"GPU-{u}"
        except Exception:
            self.index = str(device)
        self.proc, self.lines = None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------------ #
# the decode workload (LLaMA-3.2-1B shapes, W4A16, m = 1)
# ------------------------------------------------------------------------------------------------ #

def decode_bytes(layers):
    """Algorithmic HBM bytes of one decode step: packed weights, fp16 scales and zeros, bf16 x, fp32 y."""
    total = 0
    for (_, n, k) in layers:
        total += n * k // 2 + 2 * 2 * n * (k // 128) + 2 * k + 4 * n
    return total


def decode_layers(n_layers=synth.LLAMA_1B_LAYERS):
    return [(f"L{l}.{nm}", n, k) for l in range(n_layers) for (nm, n, k) in synth.LLAMA_1B_LINEARS]


def build_decode(q4, dev, seed=0):
    """Quantize the 112 weight matrices on the device (the product's quantizer) and make the inputs."""
    weights, xs, ys = [], [], []
    for (name, n, k) in decode_layers():
        W = torch.from_numpy(synth.weights((seed, "llama1b", name), n, k)).to(dev)
        weights.append(q4.q4_quantize_pack(W, 128, False))
        del W
        x = synth.activations((seed, "llama1b-decode-x", name), 1, k)
        xs.append(torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16))
        ys.append(torch.empty((1, n), dtype=torch.float32, device=dev))
    torch.cuda.synchronize()
    return weights, xs, ys


def run_decode(args, ws, rank):
    from moe_linear_layers_b200 import q4
    dev = torch.device("cuda", torch.cuda.current_device())
    layers = decode_layers()
    weights, xs, ys = build_decode(q4, dev)
    bytes_step = decode_bytes(layers)
    stream = torch.cuda.current_stream()

    def step():
        for w, x, y in zip(weights, xs, ys):
            q4.q4_linear_w4a16(x, w, y=y)

    # CUDA graph of one step (112 launches of the public call), replayed K times.
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()

    # per-launch durations of the dominant kernel (events around each launch, outside the timed region)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(weights) + 1)]
    for rep in range(3):
        ev[0].record()
        for i, (w, x, y) in enumerate(zip(weights, xs, ys)):
            q4.q4_linear_w4a16(x, w, y=y)
            ev[i + 1].record()
    torch.cuda.synchronize()
    per_launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(weights))]

    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, ws)
    ms_step = ms / args.steps
    value = ws * bytes_step * args.steps / (ms * 1e-3) / 1e9

    # end to end through the public call with host buffers: pinned x in, y back to the host
    hx = [x.cpu().pin_memory() for x in xs]
    hy = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in ys]
    h2d = sum(t.numel() * t.element_size() for t in hx)
    d2h = sum(t.numel() * t.element_size() for t in hy)

    def e2e_step():
        for hxi, x in zip(hx, xs):
            x.copy_(hxi, non_blocking=True)
        step()
        for y, hyi in zip(ys, hy):
            hyi.copy_(y, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(f0.elapsed_time(f1), ws)
    e2e_val = ws * bytes_step * args.steps / (ms_e2e * 1e-3) / 1e9

    peaks = load_peaks()
    # dominant kernel: the GEMV; achieved = algorithmic bytes of the step / step time of the graph
    roof = {"bound": "hbm", "achieved": round(value / ws, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(value / ws / peaks["hbm_gbs"], 4), "traffic": traffic_from_profiles("gemv_decode"),
            "peak_source": peaks["source"],
            "per_launch_us": {"mean": round(1e3 * float(np.mean(per_launch_ms)), 3),
                              "gate_up_8192x2048": round(1e3 * float(np.mean([per_launch_ms[i] for i, l in
                                                                               enumerate(layers) if l[0].endswith(('gate', 'up'))])), 3),
                              "kv_512x2048": round(1e3 * float(np.mean([per_launch_ms[i] for i, l in
                                                                         enumerate(layers) if l[0].endswith(('.k', '.v'))])), 3)}}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "llama-3.2-1b-shaped decode step, W4A16 GEMV m=1, 16 layers x 7 linears, "
                               "asymmetric INT4 group 128, fp32 out",
                   "linears_per_step": len(layers), "bytes_per_step": bytes_step,
                   "l2": "working set %.0f MB > 126 MB L2; no flush needed" % (bytes_step / 1e6),
                   "parallelism": f"replicas x{ws}", "launch": "CUDA graph of 112 q4_linear_w4a16 calls"},
        "roofline": roof,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "eager public-API calls, pinned host x copied in and y copied out every step"},
        "gpu_launches": len(weights) * args.steps,
        "clocks": clk.summary(),
    }
    return line


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def traffic_from_profiles(name):
    """DRAM bytes per launch recorded from an ncu capture of the current kernel (profiles/*.json), or None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(p):
        return json.load(open(p)).get(name)
    return None


# ------------------------------------------------------------------------------------------------ #
# CPU baseline: the oracle on a bounded sample of the workload
# ------------------------------------------------------------------------------------------------ #

def oracle_decode_sample(rows_per_linear=128):
    """The oracle over the first rows of layer 0's seven linears (same weights and x as the device run).
    Returns (bytes processed, seconds, threads)."""
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
    return nbytes, dt, int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline_decode():
    nbytes, dt, cores = oracle_decode_sample()
    reps = max(1, int(10.0 / max(dt, 1e-3)))
    reps = min(reps, 200)
    total_b, total_t = 0, 0.0
    for _ in range(reps):
        b, t, _ = oracle_decode_sample()
        total_b += b
        total_t += t
    return {"value": round(total_b / total_t / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} passes of the oracle over the first 128 rows of layer 0's 7 linears "
                      "(W4A16 m=1, fp64 accumulation)"}


def run_reference(args, ws, rank):
    """--impl reference: the oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_decode_sample()
    tb, tt = 0, 0.0
    for _ in range(args.steps):
        b, t, cores = oracle_decode_sample()
        tb += b
        tt += t
    v = tb / tt / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tt / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "llama-3.2-1b-shaped decode step, W4A16 GEMV m=1 (oracle sample: first 128 rows "
                                   "of layer 0's 7 linears per step)", "parallelism": "host cores"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": "first 128 rows of layer 0's 7 linears per step"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, ws, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    ws, rank, local = dist_setup()
    line = run_decode(args, ws, rank)
    if rank == 0:
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_decode()
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
