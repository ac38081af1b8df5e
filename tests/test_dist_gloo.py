"""The multi-rank host logic of bench.py, run as two gloo ranks on CPU.

With --shard replicas each rank processes its own sequence and no data
crosses ranks; with --shard heads (tests/test_dist_shard_heads.py) the ranks
split one sequence's heads.  Either way the ranks share the job's clock: the
step time is the max over ranks, and the value counts the work of the whole
job.  These tests check that logic (and the per-rank inputs) without a GPU.
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
    # heads of one sequence split over 8 ranks: the job is that one sequence
    assert abs(bench.job_value(wl, 8, 100.0, sharded=True) - one) < 1e-9
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_compressed_flops_per_sequence_and_per_head():
    """Attention FLOPs over kept rows: one count per sequence (every head
    keeps it) equals the same count repeated per head."""
    import numpy as np
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    wl = W.WORKLOADS["c3_L32K_gqa_band"]
    per_seq = np.array([25147])
    per_head = np.full((1, wl.Hq), 25147)
    a, b = bench.compressed_flops(wl, per_seq), bench.compressed_flops(wl, per_head)
    assert a == b == wl.Hq * 2.0 * wl.d * 25147 * 25148
    # heads keeping different counts
    mixed = np.arange(1, wl.Hq + 1).reshape(1, wl.Hq) * 100
    want = sum(2.0 * wl.d * n * (n + 1) for n in mixed.ravel())
    assert bench.compressed_flops(wl, mixed) == want
    # the full sequence kept gives the dense causal FLOPs
    assert bench.compressed_flops(wl, np.array([wl.L])) == bench.dense_flops(wl)


def test_both_arms_print_the_same_config():
    import argparse
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    wl = W.WORKLOADS["c4_L128K_gqa"]
    args = argparse.Namespace(tau=0.05, budget_mode="max", keep_recent=0, layout="bhld", gpus=1)
    cfg = bench.config_of(args, wl, 1)
    assert cfg["workload"] == "c4_L128K_gqa" and cfg["L"] == 131072 and cfg["parallelism"] == "single"
    assert bench.config_of(args, wl, 4)["parallelism"] == "heads4"      # the default split
    args.shard = "replicas"
    assert bench.config_of(args, wl, 4)["parallelism"] == "replicas4"


def test_stage_bytes_count_unique_kv_rows_per_group():
    """The gather's algorithmic bytes count each K/V row a KV group reads once
    (the union of its query heads' selections), per the measurement plan."""
    import sys

    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(B=1, Hq=4, Hkv=2, L=8, d=64, w=2)
    idx = torch.full((1, 4, 8), -1, dtype=torch.int32)
    sel = {0: [0, 1, 2], 1: [1, 2, 3], 2: [5, 6, 7], 3: [5, 6, 7]}   # group 0 reads 4 rows, group 1 reads 3
    for h, s in sel.items():
        idx[0, h, :3] = torch.tensor(s)
    b = bench.stage_algorithmic_bytes(wl, np.array([3]), idx)
    row = 64 * 2
    assert b["gather"] == 12 * row + 2 * 7 * row + 3 * 12 * row
    assert b["scatter"] == 4 * 8 * row + 12 * row
    assert b["score"] == 2 * 8 * row + 4 * 2 * row + 4 * 8 * 4
    # per-head counts: head 3 keeps only 2 rows, so group 1 still reads rows 5, 6, 7 (head 2)
    b2 = bench.stage_algorithmic_bytes(wl, np.array([[3, 3, 3, 2]]), idx)
    assert b2["gather"] == 11 * row + 2 * 7 * row + 3 * 11 * row
