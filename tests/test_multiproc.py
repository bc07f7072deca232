"""The benchmark's multi-process path on CPU: two gloo ranks.

With N GPUs, bench.py runs one process per GPU; each rank verifies its own
layers (weak scaling, no collective on the data path), the step time is the
slowest rank's device time, and the whole-job value counts every rank's
calls. These tests run that host logic with world_size 2 over gloo.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_env()
        assert (w, r) == (world, rank)
        # slowest rank's time, on every rank
        got = bench.max_over_ranks(10.0 + rank, "cpu")
        # each rank's own layers: distinct seeds, the same tree
        cases = bench.workload_cases("kimi", 2, rank, world)
        seeds = [c.seed for c in cases]
        trees = [c.parent.tolist() for c in cases]
        gathered = [None] * world
        dist.all_gather_object(gathered, {"seeds": seeds, "trees": trees, "max": got})
        if rank == 0:
            out.put(gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_partition_layers_and_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = out.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g["max"] for g in res] == [11.0, 11.0]
    all_seeds = res[0]["seeds"] + res[1]["seeds"]
    assert len(set(all_seeds)) == 4                    # no layer runs on two ranks
    assert res[0]["trees"][0] == res[1]["trees"][0]     # one verify step: one draft tree


def test_job_value_counts_every_rank():
    import bench
    # 61 calls per rank, 2 ranks, a 5 ms step: 10 ms of device time bought 122 calls
    assert bench.job_us_per_call(5.0, 61, 2) == pytest.approx(5000.0 / 122)
    assert bench.job_us_per_call(5.0, 61, 1) == pytest.approx(5000.0 / 61)
