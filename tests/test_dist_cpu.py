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
