"""The multi-GPU path of the benchmark is replicas: every rank runs its own layer on its own batch,
with no data-path collective; the only cross-rank steps are a barrier and the max over ranks of the
device-timed region. These run here as two gloo ranks on the CPU: the max, the whole-job throughput
built from it, and the reference arm leaving ranks other than 0 without work."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [2.5, 4.0][rank]                       # rank 1 is the slow one
        bench.barrier(world)
        m = bench.max_over_ranks(ms, world)
        value = bench.job_tokens_per_s(4096, world, m)
        # the reference arm runs on rank 0 only; other ranks return at once, before any work
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world))
        ran = None
        if rank != 0:
            import argparse
            bench.run_reference(argparse.Namespace(config="tiny", steps=3, warmup=3, gpus=world))
            ran = "returned"
        out.put((rank, m, value, ran))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_every_rank():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(world))
    for rank, m, value, ran in res:
        assert m == 4.0                                     # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 4096 / 4.0e-3)    # all ranks' tokens over that time
    assert res[1][3] == "returned"


def test_routing_stats_counts_drops():
    import numpy as np

    import bench
    st = bench.routing_stats(np.array([3, 5, 0, 8]), np.array([3, 4, 0, 6]))
    assert st == {"count_min": 0, "count_max": 8, "count_mean": 4.0, "max_over_mean": 2.0, "dropped_slots": 3}
