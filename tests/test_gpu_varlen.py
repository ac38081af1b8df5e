"""GPU parity of packed varlen batches (sequences of different lengths in one
token-major [T, H, d] tensor, offsets in cu_seqlens) against the oracle run
on every sequence alone.

Scores are compared within their tolerance; budgets, kept counts and indices
bit for bit on the GPU's own scores; outputs within the attention tolerance,
with every unselected row of every sequence exactly zero.  Equal lengths
must reproduce the batched token-major forward bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, from_dev_bf16, garbage_like, scores_close, to_dev_bf16
from test_gpu_parity import ATOL_OUT, SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu


def packed_inputs(lengths, Hq, Hkv, d, seed):
    """Seeded inputs: sequence b is the first L_b tokens of sequence b of a
    head-major workload with L = max length, packed token-major."""
    Lmax = max(max(lengths), 1)
    wl = SHAPES["gqa_d128_B2_L777_w130"].with_(B=len(lengths), Hq=Hq, Hkv=Hkv, L=Lmax, d=d, seed=seed)
    q, k, v = W.generate(wl)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    pack = lambda x: np.concatenate([x[b, :, :n].transpose(1, 0, 2) for b, n in enumerate(lengths)], axis=0)
    return pack(q), pack(k), pack(v), cu, Lmax


def run_varlen(qp, kp, vp, cu, Lmax, w, tau, mode="max", r=0):
    dq, dk, dv = (to_dev_bf16(x) for x in (qp, kp, vp))
    dcu = torch.from_numpy(cu).cuda()
    p = T.params(len(cu) - 1, qp.shape[1], kp.shape[1], Lmax, qp.shape[2], w, tau, budget_mode=mode,
                 keep_recent=r, cu_seqlens=dcu, total_tokens=qp.shape[0])
    ws = T.new_workspace(p, full=True)
    o = garbage_like(dq.shape)
    B, Hq = len(cu) - 1, qp.shape[1]
    scores = torch.empty((B, Hq, Lmax), device="cuda")
    idx = torch.empty((B, Hq, Lmax), dtype=torch.int32, device="cuda")
    kept = torch.empty((B, Hq) if mode == "per_head" else (B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, kept)
    return p, ws, o, scores, idx, kept, (dq, dk, dv, dcu)


CASES = [
    ([1000, 0, 37, 777, 1], 4, 2, 128, 48, 0.1, "max", 0),
    ([1000, 0, 37, 777, 1], 4, 2, 128, 48, 0.1, "per_head", 20),
    ([300, 129, 128, 2500], 8, 2, 64, 64, 0.2, "mean", 0),
    ([5, 700], 2, 2, 128, 130, 0.05, "per_head", 0),
]


@pytest.mark.parametrize("lengths,Hq,Hkv,d,w,tau,mode,r", CASES)
def test_varlen_forward_matches_oracle_per_sequence(lengths, Hq, Hkv, d, w, tau, mode, r):
    qp, kp, vp, cu, Lmax = packed_inputs(lengths, Hq, Hkv, d, seed=len(lengths) * 7 + d)
    p, ws, o, scores, idx, kept, _ = run_varlen(qp, kp, vp, cu, Lmax, w, tau, mode, r)
    assert_status_clean(ws)
    g_s, g_idx, g_kept = scores.cpu().numpy(), idx.cpu().numpy(), kept.cpu().numpy()
    o16 = from_dev_bf16(o)
    got_all = bf16_to_f64(o)
    G = Hq // Hkv
    for b, Lb in enumerate(lengths):
        t0 = int(cu[b])
        assert (g_idx[b, :, Lb:] == -1).all()
        if Lb == 0:
            assert (g_kept[b] == 0).all()
            continue
        hm = lambda x: np.ascontiguousarray(x[t0:t0 + Lb].transpose(1, 0, 2))[None]
        q1, k1, v1 = hm(qp), hm(kp), hm(vp)
        # scores within tolerance of the per-sequence fp64 definition
        _, s64 = O.proxy_scores(q1, k1, w, return_f64=True)
        assert scores_close(g_s[b:b + 1, :, :Lb], s64) <= 1.0
        # budget and selection bit-exact on the GPU's own scores
        kh, ks = O.coverage_budget(g_s[b:b + 1, :, :Lb], tau, mode, min(r, Lb))
        kr = O.kept_counts(kh, ks, mode)
        assert np.array_equal(g_kept[b], kh[0] if mode == "per_head" else ks[0])
        assert np.array_equal(g_idx[b:b + 1, :, :Lb], O.select_topk(g_s[b:b + 1, :, :Lb], kr, min(r, Lb)))
        # output rows of this sequence
        qc, kc, vc = O.gather_qkv(q1, k1, v1, g_idx[b:b + 1, :, :Lb], kr)
        ref = O.scatter(O.compressed_attention(qc, kc, vc, kr), g_idx[b:b + 1, :, :Lb], kr, Lb)[0]
        got = got_all[t0:t0 + Lb].transpose(1, 0, 2)
        assert np.abs(got - ref).max() <= ATOL_OUT, b
        for h in range(Hq):
            unsel = np.setdiff1d(np.arange(Lb), g_idx[b, h, :kr[0, h]])
            assert (o16[t0 + unsel, h] == 0).all()


def test_varlen_equal_lengths_equal_batched_forward():
    wl = SHAPES["gqa_d128_B2_L777_w130"]
    q, k, v = W.generate(wl)
    tm = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3))
    p_b = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, layout="blhd")
    dq, dk, dv = (to_dev_bf16(tm(x)) for x in (q, k, v))
    ws = T.new_workspace(p_b, full=True)
    o_b = garbage_like(dq.shape)
    s_b = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    i_b = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    k_b = torch.empty((wl.B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p_b, dq, dk, dv, o_b, ws, s_b, i_b, k_b)
    pk = lambda x: tm(x).reshape(wl.B * wl.L, x.shape[1], wl.d)
    cu = np.arange(wl.B + 1, dtype=np.int32) * wl.L
    _, ws2, o_v, s_v, i_v, k_v, _ = run_varlen(pk(q), pk(k), pk(v), cu, wl.L, wl.w, wl.tau)
    assert torch.equal(s_b, s_v) and torch.equal(i_b, i_v) and torch.equal(k_b, k_v)
    assert torch.equal(o_b.reshape(o_v.shape).view(torch.int16), o_v.view(torch.int16))
    assert_status_clean(ws)
    assert_status_clean(ws2)


def test_varlen_dense_and_stage_calls():
    lengths = [640, 3, 129]
    qp, kp, vp, cu, Lmax = packed_inputs(lengths, 4, 1, 128, seed=77)
    p, ws, o, scores, idx, kept, (dq, dk, dv, dcu) = run_varlen(qp, kp, vp, cu, Lmax, 32, 0.1)
    sws = T.new_workspace(p, full=False)
    # dense causal attention per sequence
    od = garbage_like(dq.shape)
    T.tsa_attend_dense(p, dq, dk, dv, od, None, sws)
    got = bf16_to_f64(od)
    for b, Lb in enumerate(lengths):
        t0 = int(cu[b])
        rows = np.unique([0, Lb // 2, Lb - 1])
        for h in (0, 3):
            ref = O.attention_rows(qp[t0:t0 + Lb, h], kp[t0:t0 + Lb, 0], vp[t0:t0 + Lb, 0], rows,
                                   O.default_scale(128))
            assert np.abs(got[t0 + rows, h] - ref).max() <= ATOL_OUT
    # stage calls reproduce the fused forward on the packed tensors
    shape = (len(lengths), 4, Lmax, 128)
    qc, kc, vc, oc = (garbage_like(shape) for _ in range(4))
    T.tsa_gather_qkv(p, dq, dk, dv, idx, kept, qc, kc, vc, sws)
    T.tsa_attend(p, qc, kc, vc, kept, oc, None, sws)
    o2 = garbage_like(dq.shape)
    T.tsa_scatter(p, oc, idx, kept, o2, sws)
    assert torch.equal(o2.view(torch.int16), o.view(torch.int16))
    o3 = garbage_like(dq.shape)
    T.tsa_attend_gathered(p, dq, dk, dv, idx, kept, o3, None, sws)
    assert torch.equal(o3.view(torch.int16), o.view(torch.int16))
    assert_status_clean(sws)


def test_varlen_out_of_range_sequence_is_flagged_and_skipped():
    """A sequence that runs past total_tokens is treated as empty (nothing of
    it is read or written) and flagged; the other sequences are unaffected."""
    lengths = [200, 50]
    qp, kp, vp, cu, Lmax = packed_inputs(lengths, 2, 2, 64, seed=5)
    bad_cu = cu.copy()
    bad_cu[2] = cu[2] + 40                       # sequence 1 claims tokens past T
    p, ws, o, scores, idx, kept, _ = run_varlen(qp, kp, vp, bad_cu, Lmax + 40, 16, 0.1)
    st, flags = T.get_device_status(ws)
    assert flags & T.DEVFLAG_BAD_INDEX
    g_kept = kept.cpu().numpy()
    assert g_kept[1] == 0
    assert (idx.cpu().numpy()[1] == -1).all()
    # the rows of sequence 1 (tokens 200..249) keep their fill pattern
    assert (o[200:250].view(torch.int16) == 0x7FC1).all().item()
    # sequence 0 as on its own
    _, ws2, o0, _, _, _, _ = run_varlen(qp[:200], kp[:200], vp[:200], cu[:2], Lmax, 16, 0.1)
    assert torch.equal(o[:200].view(torch.int16), o0.view(torch.int16))
