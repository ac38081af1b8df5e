"""GPU checks at the limits the ABI accepts and at the method's degenerate
settings.

Largest shape: L = 2^22 tokens with the largest window w = 4096.  The oracle
cannot compute 4096 x 2^22 proxy weights in reasonable time, so the scores
are checked through properties that hold at any size (each is >= 0 and they
sum to w), the budget and selection bit for bit on the GPU's own scores,
sampled output rows against the oracle, and every unselected row for exact
zeros.  Degenerate settings: tau = 0 keeps every token, so the path must
equal dense attention bit for bit; a window spanning the whole sequence;
forced keeps covering the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, garbage_like, inputs, scores_close
from test_gpu_parity import ATOL_OUT, SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu


def test_largest_length_and_window():
    wl = SHAPES["c1_mha_d64_L1024"].with_(B=1, Hq=1, Hkv=1, L=1 << 22, d=64, w=4096, tau=0.05, heavy_count=64,
                                         seed=41)
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = T.params(1, 1, 1, wl.L, 64, 4096, 0.05)
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(dq)
    scores = torch.empty((1, 1, wl.L), device="cuda")
    idx = torch.empty((1, 1, wl.L), dtype=torch.int32, device="cuda")
    ks = torch.empty((1,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, ks)
    assert T.get_device_status(ws)[0] == 0
    g_s = scores.cpu().numpy()
    assert (g_s >= 0).all()
    assert abs(g_s.astype(np.float64).sum() - 4096.0) <= 4096.0 * 1e-4
    _, ks_ref = O.coverage_budget(g_s, 0.05)
    g_idx, kb = idx.cpu().numpy(), int(ks.cpu()[0])
    assert kb == int(ks_ref[0]) and kb < wl.L
    assert np.array_equal(g_idx, O.select_topk(g_s, ks_ref))
    S = g_idx[0, 0, :kb].astype(np.int64)
    crow = np.unique(np.array([0, 1, 127, 128, kb // 2, kb - 129, kb - 2, kb - 1]))
    ref = O.attention_rows(q[0, 0][S], k[0, 0][S], v[0, 0][S], crow, O.default_scale(64))
    got = bf16_to_f64(o[0, 0, torch.from_numpy(S[crow]).cuda()])
    assert np.abs(got - ref).max() <= ATOL_OUT
    sel = torch.zeros(wl.L, dtype=torch.bool, device="cuda")
    sel[idx[0, 0, :kb].long()] = True
    nz = (o[0, 0].view(torch.int16) != 0).any(dim=-1)
    assert not (nz & ~sel).any().item()


@pytest.mark.parametrize("name", ["gqa_d128_B2_L777_w130", "gqa_d64_L2500"])
def test_tau_zero_equals_dense_attention(name):
    wl = SHAPES[name]
    _, (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, 0.0)
    ws = T.new_workspace(p, full=True)
    o, od = garbage_like(dq.shape), garbage_like(dq.shape)
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    ks = torch.empty((wl.B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, None, idx, ks)
    T.tsa_attend_dense(p, dq, dk, dv, od, None, ws)
    assert (ks == wl.L).all().item()
    assert torch.equal(idx, torch.arange(wl.L, dtype=torch.int32, device="cuda").expand_as(idx))
    assert torch.equal(o.view(torch.int16), od.view(torch.int16))
    assert_status_clean(ws)


def test_window_spans_the_sequence_and_forced_keep_all():
    wl = SHAPES["mha_d128_L129"]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    # w = L: every row is a window row; the scores sum to L
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.L, wl.tau)
    ws = T.new_workspace(p, full=True)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    T.tsa_score(p, dq, dk, scores, ws)
    _, s64 = O.proxy_scores(q, k, wl.L, return_f64=True)
    assert scores_close(scores.cpu().numpy(), s64) <= 1.0   # element-wise 1e-5 relative
    assert np.allclose(scores.cpu().numpy().sum(axis=-1), wl.L, rtol=1e-5)
    # keep_recent = L keeps every token: the dense result
    p2 = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, 0.5, keep_recent=wl.L)
    ws2 = T.new_workspace(p2, full=True)
    o, od = garbage_like(dq.shape), garbage_like(dq.shape)
    T.tsa_forward(p2, dq, dk, dv, o, ws2)
    T.tsa_attend_dense(p2, dq, dk, dv, od, None, ws2)
    assert torch.equal(o.view(torch.int16), od.view(torch.int16))
    assert_status_clean(ws)
    assert_status_clean(ws2)
