"""GPU parity of the budget modes (max, mean, per-head) and of forced keeps of
the most recent tokens, against the oracle.

Budget, selection and the kept counts are integer results and must match the
oracle bit for bit; outputs are compared within the attention tolerance on
every row at small sizes and on sampled rows at the 32K workload, with the
unselected rows checked to be exactly zero everywhere.
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, from_dev_bf16, garbage_like, inputs
from test_gpu_full_configs import sample_rows
from test_gpu_parity import ATOL_OUT, SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu

MODES = [("max", 0), ("max", 37), ("mean", 0), ("mean", 5), ("per_head", 0), ("per_head", 64)]


def Pm(wl, mode, r, tau=None):
    return T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau if tau is None else tau,
                    budget_mode=mode, keep_recent=min(r, wl.L))


def kept_buffer(wl, mode):
    shape = (wl.B, wl.Hq) if mode == "per_head" else (wl.B,)
    return torch.full(shape, -7, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("mode,r", MODES)
@pytest.mark.parametrize("name", ["gqa_d128_B2_L777_w130", "gqa_d64_L2500", "single_token"])
def test_budget_select_modes_bit_exact(name, mode, r):
    wl = SHAPES[name]
    r = min(r, wl.L)
    q, k, _ = W.generate(wl)
    s32 = O.proxy_scores(q, k, wl.w)           # the oracle's fp32 scores feed both sides
    k_head, k_seq = O.coverage_budget(s32, wl.tau, mode, r)
    idx = O.select_topk(s32, O.kept_counts(k_head, k_seq, mode), r)
    p = Pm(wl, mode, r)
    ws = T.new_workspace(p, full=False)
    ds = torch.from_numpy(s32).cuda()
    g_kh = torch.full((wl.B, wl.Hq), -7, dtype=torch.int32, device="cuda")
    g_ks = torch.full((wl.B,), -7, dtype=torch.int32, device="cuda")
    g_idx = torch.full((wl.B, wl.Hq, wl.L), -7, dtype=torch.int32, device="cuda")
    T.tsa_budget(p, ds, g_kh, g_ks, ws)
    T.tsa_select(p, ds, g_kh if mode == "per_head" else g_ks, g_idx, ws)
    assert np.array_equal(g_kh.cpu().numpy(), k_head)
    assert np.array_equal(g_ks.cpu().numpy(), k_seq)
    assert np.array_equal(g_idx.cpu().numpy(), idx)
    assert_status_clean(ws)


def test_budget_modes_golden_fixtures():
    import test_oracle_budget_modes as pins
    for ex in pins._mode_examples():
        s = np.array([ex["heads"]], dtype=np.float32)
        H, L = s.shape[1], s.shape[2]
        p = T.params(1, H, 1, L, 64, 1, ex["tau"], budget_mode=ex["mode"], keep_recent=ex["keep_recent"])
        ws = T.new_workspace(p, full=False)
        kh = torch.empty((1, H), dtype=torch.int32, device="cuda")
        ks = torch.empty((1,), dtype=torch.int32, device="cuda")
        ix = torch.empty((1, H, L), dtype=torch.int32, device="cuda")
        ds = torch.from_numpy(s).cuda()
        T.tsa_budget(p, ds, kh, ks, ws)
        T.tsa_select(p, ds, kh if ex["mode"] == "per_head" else ks, ix, ws)
        assert list(kh.cpu().numpy()[0]) == ex["k_head"], ex["name"]
        assert int(ks.cpu()[0]) == ex["k_seq"], ex["name"]
        for h, want in enumerate(ex["idx"]):
            n = ex["kept"][h]
            assert list(ix.cpu().numpy()[0, h, :n]) == want, ex["name"]
            assert (ix.cpu().numpy()[0, h, n:] == -1).all(), ex["name"]


def _check_forward(wl, mode, r, q, k, v, o, scores, idx, kept, rows_of=None):
    g_s, g_idx, g_kept = scores.cpu().numpy(), idx.cpu().numpy(), kept.cpu().numpy()
    # budget and selection are exactly the oracle's on the GPU's own scores
    kh, ks = O.coverage_budget(g_s, wl.tau, mode, r)
    kept_ref = O.kept_counts(kh, ks, mode)
    assert np.array_equal(g_kept, kh if mode == "per_head" else ks)
    assert np.array_equal(g_idx, O.select_topk(g_s, kept_ref, r))
    if r:
        for b in range(wl.B):
            for h in range(wl.Hq):
                assert set(range(wl.L - r, wl.L)) <= set(g_idx[b, h, :kept_ref[b, h]].tolist())
    # unselected rows exactly zero
    o16 = from_dev_bf16(o)
    for b in range(wl.B):
        for h in range(wl.Hq):
            unsel = np.setdiff1d(np.arange(wl.L), g_idx[b, h, :kept_ref[b, h]])
            assert (o16[b, h, unsel] == 0).all()
    # output rows against the oracle over the GPU's selection
    if rows_of is None:
        qc, kc, vc = O.gather_qkv(q, k, v, g_idx, kept_ref)
        ref = O.scatter(O.compressed_attention(qc, kc, vc, kept_ref), g_idx, kept_ref, wl.L)
        assert np.abs(bf16_to_f64(o) - ref).max() <= ATOL_OUT
    else:
        for b, h, rows in rows_of:
            ref = O.output_rows(q, k, v, g_idx, kept_ref, b, h, rows)
            got = bf16_to_f64(o[b, h, torch.from_numpy(rows).cuda()])
            assert np.abs(got - ref).max() <= ATOL_OUT, (b, h)
    return kept_ref


@pytest.mark.parametrize("mode,r", MODES)
@pytest.mark.parametrize("name", ["gqa_d128_B2_L777_w130", "gqa_d64_L2500", "mha_d128_L129"])
def test_forward_modes(name, mode, r):
    wl = SHAPES[name]
    r = min(r, wl.L)
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = Pm(wl, mode, r)
    ws = T.new_workspace(p, full=True)
    o = garbage_like(dq.shape)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    kept = kept_buffer(wl, mode)
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, kept)
    kept_ref = _check_forward(wl, mode, r, q, k, v, o, scores, idx, kept)
    if mode == "per_head" and r == 0 and wl.Hq >= 4:
        assert len(set(kept_ref.ravel().tolist())) > 1     # heads really keep different counts
    assert_status_clean(ws)


@pytest.mark.parametrize("mode,r", [("per_head", 0), ("mean", 16)])
def test_stage_calls_equal_forward_bit_for_bit(mode, r):
    """gather -> attend -> scatter with per-head or mean counts reproduces the
    fused forward exactly (the same kernels, the same arithmetic)."""
    wl = SHAPES["gqa_d128_B2_L777_w130"]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = Pm(wl, mode, r)
    ws = T.new_workspace(p, full=True)
    o = garbage_like(dq.shape)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    kept = kept_buffer(wl, mode)
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, kept)
    sws = T.new_workspace(p, full=False)
    qc, kc, vc, oc = (garbage_like(dq.shape) for _ in range(4))
    T.tsa_gather_qkv(p, dq, dk, dv, idx, kept, qc, kc, vc, sws)
    T.tsa_attend(p, qc, kc, vc, kept, oc, None, sws)
    o2 = garbage_like(dq.shape)
    T.tsa_scatter(p, oc, idx, kept, o2, sws)
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))
    assert_status_clean(sws)


@pytest.mark.parametrize("mode,r", [("per_head", 0), ("mean", 256), ("per_head", 1024)])
def test_forward_modes_32k_sampled(mode, r):
    wl = W.WORKLOADS["c3_L32K_gqa_band"]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = Pm(wl, mode, r)
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(dq)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    kept = kept_buffer(wl, mode)
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, kept)
    assert T.get_device_status(ws)[0] == 0
    rng = np.random.default_rng(5)
    rows_of = [(0, h, sample_rows(wl.L, rng, n=8)) for h in (0, 13, wl.Hq - 1)]
    _check_forward(wl, mode, r, q, k, v, o, scores, idx, kept, rows_of)
