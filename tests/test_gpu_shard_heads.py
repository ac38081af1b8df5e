"""GPU check of the head-sharded forward (tsa_forward_begin / tsa_forward_end).

The query heads of each sequence are split as shard_heads splits them over
2 and 4 devices.  On this one GPU the "devices" run one after another: each
runs tsa_forward_begin on its own contiguous head slice, the B budget
partials are combined on the device with the op budget_reduce_op names (the
place of the all-reduce; nothing waits on another launch), and each runs
tsa_forward_end.  Every shard must reproduce, bit for bit, the slice of its
heads of the single-call tsa_forward on all heads -- scores, per-head counts,
budget, indices and output -- in every budget mode; the budget also equals
the oracle's on the GPU's scores.
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import inputs
from test_gpu_parity import assert_status_clean

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS["c1_L1K_mha_d64"].with_(B=2, Hq=8, Hkv=2, L=1000, d=128, w=64, tau=0.1, heavy_count=8,
                                         seed=51)


def _full(p, dq, dk, dv, wl):
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(dq)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    kshape = (wl.B, wl.Hq) if p.budget_mode == T.BUDGET_PER_HEAD else (wl.B,)
    kept = torch.empty(kshape, dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, kept)
    assert_status_clean(ws)
    return o, scores, idx, kept


@pytest.mark.parametrize("mode", ["max", "mean", "per_head"])
@pytest.mark.parametrize("world", [1, 2, 4])
def test_sharded_halves_reproduce_the_whole_forward(mode, world):
    wl = WL
    _, (dq, dk, dv) = inputs(wl)
    p_all = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, budget_mode=mode)
    o_ref, s_ref, idx_ref, kept_ref = _full(p_all, dq, dk, dv, wl)
    shards = []
    for r in range(world):
        h0, h1, kv0, kv1 = T.shard_heads(wl.Hq, wl.Hkv, world, r)
        q, k, v = (x.contiguous() for x in (dq[:, h0:h1], dk[:, kv0:kv1], dv[:, kv0:kv1]))
        p = T.params(wl.B, h1 - h0, kv1 - kv0, wl.L, wl.d, wl.w, wl.tau, budget_mode=mode)
        ws = T.new_workspace(p, full=True)
        scores = torch.empty((wl.B, h1 - h0, wl.L), device="cuda")
        k_head = torch.empty((wl.B, h1 - h0), dtype=torch.int32, device="cuda")
        k_part = torch.full((wl.B,), -1, dtype=torch.int32, device="cuda")
        T.tsa_forward_begin(p, q, k, k_part, ws, scores_out=scores, k_head_out=k_head)
        shards.append(dict(h=(h0, h1), p=p, q=q, k=k, v=v, ws=ws, scores=scores, k_head=k_head, k_part=k_part))
    op = T.budget_reduce_op(mode)
    parts = torch.stack([s["k_part"] for s in shards])
    reduced = parts.max(0).values if op == "max" else parts.sum(0, dtype=torch.int32)   # the all-reduce
    for s in shards:
        h0, h1 = s["h"]
        o = torch.empty_like(s["q"])
        idx = torch.empty((wl.B, h1 - h0, wl.L), dtype=torch.int32, device="cuda")
        kept = torch.empty((wl.B, h1 - h0) if mode == "per_head" else (wl.B,), dtype=torch.int32, device="cuda")
        T.tsa_forward_end(s["p"], wl.Hq, s["q"], s["k"], s["v"], o, None if op is None else reduced, s["ws"],
                          scores=s["scores"], k_head=s["k_head"], idx_out=idx, k_seq_out=kept)
        assert_status_clean(s["ws"])
        assert torch.equal(s["scores"].view(torch.int32), s_ref[:, h0:h1].view(torch.int32))
        if mode == "per_head":
            assert torch.equal(kept, kept_ref[:, h0:h1])
        else:
            assert torch.equal(kept, kept_ref)
        assert torch.equal(idx, idx_ref[:, h0:h1])
        assert torch.equal(o.view(torch.int16), o_ref[:, h0:h1].view(torch.int16))
    # the combined budget is the oracle's, computed from the GPU's scores of all heads
    _, ks = O.coverage_budget(s_ref.cpu().numpy(), wl.tau, mode)
    if mode != "per_head":
        assert np.array_equal(kept_ref.cpu().numpy(), ks)


def test_forward_sharded_on_one_device_equals_tsa_forward():
    """The binding's helper without a process group: begin, no exchange, end."""
    wl = WL
    _, (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    o_ref, _, idx_ref, kept_ref = _full(p, dq, dk, dv, wl)
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(dq)
    idx = torch.empty_like(idx_ref)
    kept = torch.empty_like(kept_ref)
    T.forward_sharded(p, wl.Hq, dq, dk, dv, o, ws, idx_out=idx, k_seq_out=kept)
    assert_status_clean(ws)
    assert torch.equal(kept, kept_ref) and torch.equal(idx, idx_ref)
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))


def test_end_rejects_bad_arguments_before_any_work():
    wl = WL
    _, (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(dq)
    red = torch.full((wl.B,), wl.L, dtype=torch.int32, device="cuda")
    with pytest.raises(T.TSAError) as e:                        # fewer heads in all than here
        T.tsa_forward_end(p, wl.Hq - 1, dq, dk, dv, o, red, ws)
    assert e.value.status == 1
    with pytest.raises(T.TSAError) as e:                        # MAX mode needs the reduced budget
        T.tsa_forward_end(p, wl.Hq, dq, dk, dv, o, None, ws)
    assert e.value.status == 1
