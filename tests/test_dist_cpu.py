"""Multi-rank host logic of bench.py on CPU with two gloo ranks: each rank
gets its own seeded batch (token sharding, weak scaling), the timed total is
the max over ranks, and the reported rate counts every rank's tokens."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from quantized_linear_token_b200 import workloads as W
        wl = W.WORKLOADS["dit_image"]
        x = bench.rank_batch(wl, 3072, 8, rank)
        local_ms = 10.0 + 5.0 * rank           # the slower rank decides
        mx = bench.max_over_ranks(local_ms)
        out[rank] = (x.tobytes(), mx, bench.whole_job_rate(world, 8, 3, mx))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_tokens_and_time_by_the_slowest():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    x0, m0, v0 = out[0]
    x1, m1, v1 = out[1]
    assert x0 != x1                              # each rank has its own batch
    assert m0 == m1 == 15.0                      # max over ranks
    assert v0 == v1 == pytest.approx(2 * 8 * 3 / 15e-3)


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(1, 100, 2, 10.0) == pytest.approx(20000.0)


def test_both_arms_report_the_same_workload_config():
    # the reference arm and this arm describe a run by the same config keys
    import argparse

    import bench
    from quantized_linear_token_b200 import workloads as W
    for key in ("dit_image", "dit_mlp", "video_dit", "stress"):
        wl = W.WORKLOADS[key]
        for lay in wl.layers:
            args = argparse.Namespace(workload=key, layer=lay.name, tokens=0, gpus=2)
            cfg = bench.workload_config(args, wl, lay, wl.tokens, 2)
            assert cfg["layer"] == lay.name and cfg["tokens_per_gpu"] == wl.tokens
            assert cfg["h"] == lay.d_in & -lay.d_in and cfg["x_dtype"] == "bf16"
            assert cfg["parallelism"].startswith("token-sharded x2")


def test_clock_sampler_summary_from_nvidia_smi_lines():
    # the nvidia-smi fallback: median SM clock of the parsed samples, the
    # highest power, and every throttle reason active in any sample
    import bench

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs = bench.ClockSampler("GPU-test")
    cs.proc = _Proc()
    cs.lines = [
        "0, 1965, 1965, 250.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 1001.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1300, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    out = cs.stop()
    assert out["sm_max_mhz"] == 1965.0 and out["samples"] == 4
    assert out["sm_mhz"] == 1750.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == 1001.0
    assert bench.ClockSampler("GPU-test").stop()["reasons"] == ["nvidia-smi unavailable"]


def test_nvml_clock_sampler_keeps_the_timed_region(monkeypatch):
    # NVML sampling with host timestamps: the summary covers only samples taken
    # inside the timed region, and reasons are decoded from the event mask
    import sys
    import time
    import types

    import bench

    state = {"i": 0}
    clocks = [1965, 1965, 1500, 1450, 1480, 1965]
    masks = [0, 0, 0x4, 0x4 | 0x40, 0x4, 0]

    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda uuid: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetPowerUsage=lambda h: 900000,
    )

    def clock(h, kind):
        state["i"] += 1
        return clocks[min(state["i"] - 1, len(clocks) - 1)]

    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: masks[min(state["i"] - 1, len(masks) - 1)]
    monkeypatch.setitem(sys.modules, "pynvml", fake)

    c = bench.start_clock_sampler("GPU-test")
    assert isinstance(c, bench.NvmlClockSampler)
    c.stop_flag.set()                       # drive the samples by hand instead of the thread
    c.thread.join()
    c.samples = []
    t = time.perf_counter()
    for k in range(6):
        c.samples.append((t + k, float(clocks[k]), masks[k], 900.0))
    out = bench.stop_clock_sampler(c, t + 2, t + 4)
    assert out["samples"] == 3 and out["sm_mhz"] == 1480.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert out["source"] == "NVML, timed region"
    out = bench.stop_clock_sampler(c, t + 10, t + 10.001)   # no sample inside: the nearest ones
    assert out["samples"] == 3 and out["source"].startswith("NVML, the samples nearest")


def test_clock_sampler_falls_back_to_nvidia_smi(monkeypatch):
    import sys
    import types

    import bench

    def boom():
        raise RuntimeError("no NVML here")

    monkeypatch.setitem(sys.modules, "pynvml", types.SimpleNamespace(nvmlInit=boom))
    c = bench.start_clock_sampler("GPU-test")
    assert isinstance(c, bench.ClockSampler)
    out = bench.stop_clock_sampler(c, 0.0, 1.0)
    assert "samples" in out


def test_nvml_clock_sampler_thread_polls(monkeypatch):
    import sys
    import time
    import types

    import bench

    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1, nvmlInit=lambda: None, nvmlDeviceGetHandleByUUID=lambda uuid: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965, nvmlDeviceGetPowerUsage=lambda h: 500000,
        nvmlDeviceGetClockInfo=lambda h, kind: 1700,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.start_clock_sampler("GPU-test")
    t0 = time.perf_counter()
    time.sleep(0.03)
    t1 = time.perf_counter()
    out = bench.stop_clock_sampler(c, t0, t1)
    assert out["samples"] >= 3 and out["sm_mhz"] == 1700.0 and out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == 500.0 and not c.thread.is_alive()
