"""Head-sharded forward, host logic on CPU (gloo, world size 2).

When the query heads of one sequence are split over devices, every step of
the method is per head except the budget, which [GS] "Cobertura Dinamica de
Tokens" makes global across a sequence's heads.  The library splits the
forward around that one exchange (tsa_forward_begin / tsa_forward_end); the
binding's helpers say which heads a device holds (shard_heads) and how the
B budget partials combine (budget_reduce_op).  Here each gloo rank runs the
oracle on its own heads, combines the partials with a real all-reduce using
the product's reduce op, finishes the budget the way tsa_forward_end does,
and must reproduce the single-process oracle exactly: the same k_b, the same
indices and the same outputs for its heads, in every budget mode.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WL = W.WORKLOADS["c1_L1K_mha_d64"].with_(B=2, Hq=8, Hkv=2, L=96, d=64, w=16, tau=0.2, heavy_count=4,
                                         seed=41)
MODES = ("max", "mean", "per_head")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_forward(q, k, v, wl, world, rank, mode, reduce_fn):
    """This rank's heads through the oracle: scores and per-head counts, the
    budget partial, `reduce_fn` over the ranks, the budget, then steps 3-6."""
    h0, h1, kv0, kv1 = T.shard_heads(wl.Hq, wl.Hkv, world, rank)
    ql, kl, vl = q[:, h0:h1], k[:, kv0:kv1], v[:, kv0:kv1]
    scores = O.proxy_scores(ql, kl, wl.w)
    k_head, _ = O.coverage_budget(scores, wl.tau, mode)
    op = T.budget_reduce_op(mode)
    if op == "max":
        part = k_head.max(axis=1)
    elif op == "sum":
        part = k_head.astype(np.int64).sum(axis=1)
    else:
        part = None
    red = reduce_fn(part, op) if op is not None else None
    if mode == "max":
        kept = O.kept_counts(k_head, red.astype(np.int32), "max")
        k_seq = red.astype(np.int32)
    elif mode == "mean":
        k_seq = (-(-red // wl.Hq)).astype(np.int32)          # ceil(sum / Hq_total), as tsa_forward_end
        kept = O.kept_counts(k_head, k_seq, "mean")
    else:
        kept = k_head
        k_seq = None
    idx = O.select_topk(scores, kept)
    qc, kc, vc = O.gather_qkv(ql, kl, vl, idx, kept)
    o = O.scatter(O.compressed_attention(qc, kc, vc, kept), idx, kept, wl.L)
    return dict(h=(h0, h1), k_head=k_head, k_seq=k_seq, idx=idx, o=o)


def _worker(rank, world, port, out):
    import datetime
    import sys

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = W.generate(WL)

        def reduce_fn(part, op):
            t = torch.from_numpy(np.ascontiguousarray(part, dtype=np.int64))
            dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
            return t.numpy()

        res = {m: _local_forward(q, k, v, WL, world, rank, m, reduce_fn) for m in MODES}
        out.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _check_against_single_process(results):
    q, k, v = W.generate(WL)
    for mode in MODES:
        ref = O.forward(q, k, v, WL.w, WL.tau, mode=mode)
        heads = []
        for r in results:
            got = r[mode]
            h0, h1 = got["h"]
            heads += list(range(h0, h1))
            assert np.array_equal(got["k_head"], ref["k_head"][:, h0:h1]), mode
            if got["k_seq"] is not None:
                assert np.array_equal(got["k_seq"], ref["k_seq"]), mode
            assert np.array_equal(got["idx"], ref["idx"][:, h0:h1]), mode
            assert np.array_equal(got["o"], ref["o"][:, h0:h1]), mode
        assert heads == list(range(WL.Hq))


def test_two_gloo_ranks_reproduce_the_single_process_oracle():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    _check_against_single_process([res[r] for r in range(world)])


@pytest.mark.parametrize("world", [1, 4, 8])
def test_any_even_split_reproduces_the_single_process_oracle(world):
    """The same pipeline with the all-reduce done in numpy: 8 query heads over
    4 devices (each holds half a GQA group, its KV head shared) and over 8
    (one query head each)."""
    q, k, v = W.generate(WL)
    parts = {}

    def first_pass(part, op):
        parts.setdefault(op, []).append(part)
        return part

    for r in range(world):
        for m in MODES:
            _local_forward(q, k, v, WL, world, r, m, first_pass)
    reduced = {op: (np.max(ps, axis=0) if op == "max" else np.sum(ps, axis=0)) for op, ps in parts.items()}
    results = [{m: _local_forward(q, k, v, WL, world, r, m, lambda part, op: reduced[op]) for m in MODES}
               for r in range(world)]
    _check_against_single_process(results)


def test_shard_heads_partitions_heads_and_keeps_gqa_groups_whole():
    for Hq, Hkv, world in [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8), (32, 8, 16), (32, 8, 32),
                           (28, 4, 2), (28, 4, 4), (28, 4, 28), (4, 4, 4), (6, 2, 2), (6, 2, 6)]:
        G = Hq // Hkv
        seen = []
        for r in range(world):
            h0, h1, kv0, kv1 = T.shard_heads(Hq, Hkv, world, r)
            assert h1 - h0 == Hq // world
            seen += list(range(h0, h1))
            # every local query head reads a local KV head, in the local grouping
            n_kv = kv1 - kv0
            assert n_kv >= 1 and (h1 - h0) % n_kv == 0
            g_local = (h1 - h0) // n_kv
            for h in range(h0, h1):
                assert h // G == kv0 + (h - h0) // g_local
        assert seen == list(range(Hq))
    # 4 heads per device across 7-head groups, 2 per device across 3-head groups, splits that do not
    # divide, and a rank outside the world
    for bad in [(28, 4, 7, 0), (6, 2, 3, 0), (12, 3, 2, 0), (32, 8, 3, 0), (32, 8, 64, 0), (32, 8, 2, 2),
                (30, 4, 2, 0)]:
        with pytest.raises(ValueError):
            T.shard_heads(*bad)


def test_budget_reduce_op_per_mode():
    assert T.budget_reduce_op("max") == "max" and T.budget_reduce_op(T.BUDGET_MAX) == "max"
    assert T.budget_reduce_op("mean") == "sum" and T.budget_reduce_op(T.BUDGET_MEAN) == "sum"
    assert T.budget_reduce_op("per_head") is None and T.budget_reduce_op(T.BUDGET_PER_HEAD) is None
