"""Host logic of the multi-GPU bench path on CPU: two gloo ranks, max-over-ranks timing and the
whole-job value (every rank runs an independent replica of the decode step)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                # each rank's own timing
        m = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        out[rank] = m
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()   # no fork of this threaded process
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 15.0


def test_decode_bytes_per_step():
    layers = bench.decode_layers()
    assert len(layers) == 112
    # packed weights alone: 16 layers x 60.8M codes / 2 bytes
    assert sum(n * k for (_, n, k) in layers) // 2 == 486539264
    b = bench.decode_bytes(layers)
    assert 0.5e9 < b < 0.53e9


def test_small_m_attainable_bound(monkeypatch):
    """The bound a small-m GEMM's bytes set: min(tensor peak, HBM bandwidth x ops per byte)."""
    monkeypatch.setattr(bench, "load_peaks", lambda: {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0,
                                                      "bf16_tflops_sustained": 1400.0, "source": "test"})
    layers = bench.decode_layers()
    ops = 2 * 64 * sum(n * k for (_, n, k) in layers)
    r = bench.with_attainable({"value": 50.0, "roofline": {"peak": 1400.0}}, 64, False)
    rf = r["roofline"]
    wbytes = sum(n * k // 2 + n * (k // 128) * 4 for (_, n, k) in layers)
    abytes = sum(64 * k * 2 + 2 * 64 * n for (_, n, k) in layers)
    assert rf["bytes_per_step"] == wbytes + abytes
    assert abs(rf["attainable"] - min(1400.0, 6000.0 * ops / (wbytes + abytes) / 1e3)) < 0.1
    assert rf["bound_at_this_m"] == "hbm" and abs(rf["frac_of_attainable"] - 50.0 / rf["attainable"]) < 1e-3
    big = bench.with_attainable({"value": 700.0, "roofline": {"peak": 1400.0}}, 4096, False)["roofline"]
    assert big["bound_at_this_m"] == "tensor" and big["attainable"] == 1400.0


def test_moe_hotness_tiers_cover_the_experts():
    tiers = bench.MOE_TIERS
    assert tiers[0][0] == 0 and tiers[-1][1] == bench.MOE["E"]
    assert all(a[1] == b[0] for a, b in zip(tiers, tiers[1:]))
    assert [t[2] for t in tiers] == [32, 64, 128]          # hot, ordinary, cold


def test_memory_footprint_closed_form():
    """Every decode-step k is a multiple of 128, so per weight the INT4 layout holds half a byte of code
    plus 2 (sym) or 4 (asym) bytes of fp16 scale and zero per 128 weights, against 2 bytes of fp16."""
    f = bench.footprint(bench.decode_layers())
    assert f["int4_asym_g128_bytes"] / f["fp16_bytes"] == (0.5 + 4 / 128) / 2 == 0.265625
    assert f["int4_sym_g128_bytes"] / f["fp16_bytes"] == (0.5 + 2 / 128) / 2 == 0.2578125
    assert f["ratio_asym_g128"] == 0.2656 and f["ratio_sym_g128"] == 0.2578


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The clock record the bench line carries: the median SM clock of the samples, the throttle reasons
    seen (NVML's bitmask mapped to names), the highest power; and an 'unavailable' record without NVML.
    The fake only answers reads, as the real sampler only reads."""
    import sys
    import time
    import types

    clocks = iter([1965, 1965, 1800] + [1965] * 10000)
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda u: "gpu0"
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    nv.nvmlDeviceGetClockInfo = lambda h, c: next(clocks)
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 | 0x1   # power cap and an unnamed bit
    nv.nvmlDeviceGetPowerUsage = lambda h: 712_300                    # mW
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: types.SimpleNamespace(uuid="1234"))
    with bench.ClockSampler(0, period_s=0.001) as cs:
        time.sleep(0.05)
    s = cs.summary()
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["samples"] >= 3
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 712.3

    monkeypatch.setitem(sys.modules, "pynvml", None)                  # import fails: no NVML
    with bench.ClockSampler(0) as cs:
        pass
    assert cs.summary()["reasons"] == ["unavailable"] and cs.summary()["samples"] == 0


def test_traffic_figure_is_dropped_when_its_kernel_source_changes(tmp_path, monkeypatch):
    """profiles/traffic.txt keys each ncu DRAM figure to the SHA-256 of the kernel source it was captured
    from: the bench reports it while the source is unchanged and null once it differs."""
    import hashlib
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "kern.cu"
    src.write_text("__global__ void k() {}\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "traffic.txt").write_text(f"k_launch 123456 {digest} kern.cu\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("k_launch") == 123456
    assert bench.traffic_from_profiles("other") is None
    src.write_text("__global__ void k() { }\n")
    assert bench.traffic_from_profiles("k_launch") is None
