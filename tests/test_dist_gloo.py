"""The multi-rank host logic of bench.py, run as two gloo ranks on CPU.

The path shards by sequence: each rank processes its own sequence and no data
crosses ranks.  What the ranks share is the job's clock: the step time is the
max over ranks and the value sums every rank's work.  These tests check that
logic (and the per-rank inputs) without a GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import workloads as W

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
        wl = bench.rank_workload(W.WORKLOADS["c1_L1K_mha_d64"].with_(L=64), rank)
        q, _, _ = W.generate(wl)
        out.put((rank, t, wl.seed, int(q[0, 0, 0, 0])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_ranks_share_clock_not_data(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(out.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [10.0 + world - 1] * world        # max over ranks everywhere
    assert len({r[2] for r in res}) == world                         # distinct per-rank seeds
    assert len({r[3] for r in res}) == world                         # hence distinct inputs


def test_job_value_sums_ranks():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    wl = W.WORKLOADS["c4_L128K_gqa"]
    one = bench.job_value(wl, 1, 100.0)
    assert abs(one - bench.dense_flops(wl) / 0.1 / 1e12) < 1e-9
    assert abs(bench.job_value(wl, 8, 100.0) - 8 * one) < 1e-6
    assert bench.max_over_ranks(3.5, None, None) == 3.5
