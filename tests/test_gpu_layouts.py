"""GPU parity of the token-major layout ([B, L, H, d] q, k, v, o; the layout a
prefill engine's projections produce) against the head-major one and the
oracle.

The layout changes only how rows are addressed, so every stage on the same
seeded inputs must give bit-identical scores, budgets, indices, compressed
tensors and outputs in both layouts; the token-major output is also compared
with the oracle directly (on every row at small sizes, on sampled rows at the
32K workload).
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, garbage_like, inputs
from test_gpu_full_configs import sample_rows
from test_gpu_parity import ATOL_OUT, SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu

NAMES = ["gqa_d128_B2_L777_w130", "gqa_d64_L2500", "mha_d128_L129", "single_token"]


def tok_major(t):
    """[B, H, L, d] -> contiguous [B, L, H, d] (a copy; no arithmetic)."""
    return t.transpose(1, 2).contiguous()


def head_major(t):
    return t.transpose(1, 2).contiguous()


def run_forward(wl, p, q, k, v, out_shape, mode="max"):
    ws = T.new_workspace(p, full=True)
    o = garbage_like(out_shape)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    kept = torch.empty((wl.B, wl.Hq) if mode == "per_head" else (wl.B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, q, k, v, o, ws, scores, idx, kept)
    assert_status_clean(ws)
    return o, scores, idx, kept


@pytest.mark.parametrize("mode", ["max", "per_head"])
@pytest.mark.parametrize("name", NAMES)
def test_forward_token_major_equals_head_major_and_oracle(name, mode):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p_h = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, budget_mode=mode)
    p_t = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, budget_mode=mode, layout="blhd")
    o_h, s_h, i_h, k_h = run_forward(wl, p_h, dq, dk, dv, dq.shape, mode)
    tq, tk, tv = tok_major(dq), tok_major(dk), tok_major(dv)
    o_t, s_t, i_t, k_t = run_forward(wl, p_t, tq, tk, tv, tq.shape, mode)
    assert torch.equal(s_h, s_t) and torch.equal(i_h, i_t) and torch.equal(k_h, k_t)
    assert torch.equal(head_major(o_t).view(torch.int16), o_h.view(torch.int16))
    # the token-major output against the oracle over the GPU's selection
    g_s, g_idx = s_t.cpu().numpy(), i_t.cpu().numpy()
    kh, ks = O.coverage_budget(g_s, wl.tau, mode)
    kept = O.kept_counts(kh, ks, mode)
    assert np.array_equal(g_idx, O.select_topk(g_s, kept))
    qc, kc, vc = O.gather_qkv(q, k, v, g_idx, kept)
    ref = O.scatter(O.compressed_attention(qc, kc, vc, kept), g_idx, kept, wl.L)
    got = bf16_to_f64(o_t).transpose(0, 2, 1, 3)
    assert np.abs(got - ref).max() <= ATOL_OUT


@pytest.mark.parametrize("name", ["gqa_d128_B2_L777_w130", "gqa_d64_L2500"])
def test_stage_calls_token_major(name):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p_h = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    p_t = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, layout="blhd")
    tq, tk, tv = tok_major(dq), tok_major(dk), tok_major(dv)
    ws_h, ws_t = T.new_workspace(p_h, full=False), T.new_workspace(p_t, full=False)
    # scores
    s_h = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    s_t = torch.empty_like(s_h)
    T.tsa_score(p_h, dq, dk, s_h, ws_h)
    T.tsa_score(p_t, tq, tk, s_t, ws_t)
    assert torch.equal(s_h, s_t)
    kh = torch.empty((wl.B, wl.Hq), dtype=torch.int32, device="cuda")
    ks = torch.empty((wl.B,), dtype=torch.int32, device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    T.tsa_budget(p_h, s_h, kh, ks, ws_h)
    T.tsa_select(p_h, s_h, ks, idx, ws_h)
    # gather from the token-major tensors gives the same compressed buffers
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    c_h = [garbage_like(shape) for _ in range(3)]
    c_t = [garbage_like(shape) for _ in range(3)]
    T.tsa_gather_qkv(p_h, dq, dk, dv, idx, ks, *c_h, ws_h)
    T.tsa_gather_qkv(p_t, tq, tk, tv, idx, ks, *c_t, ws_t)
    ks_np = ks.cpu().numpy()
    for a, b in zip(c_h, c_t):
        for bb in range(wl.B):
            n = int(ks_np[bb])
            assert torch.equal(a[bb, :, :n].view(torch.int16), b[bb, :, :n].view(torch.int16))
    # attention + scatter epilogue writes the token-major output in place
    o_h, o_t = garbage_like(dq.shape), garbage_like(tq.shape)
    T.tsa_attend_scatter(p_h, *c_h, idx, ks, o_h, None, ws_h)
    T.tsa_attend_scatter(p_t, *c_t, idx, ks, o_t, None, ws_t)
    assert torch.equal(head_major(o_t).view(torch.int16), o_h.view(torch.int16))
    # compressed attention + plain scatter into the token-major output
    oc = garbage_like(shape)
    T.tsa_attend(p_t, *c_t, ks, oc, None, ws_t)
    o2 = garbage_like(tq.shape)
    T.tsa_scatter(p_t, oc, idx, ks, o2, ws_t)
    assert torch.equal(o2.view(torch.int16), o_t.view(torch.int16))
    # fully gathering attention straight from the token-major tensors
    o3 = garbage_like(tq.shape)
    T.tsa_attend_gathered(p_t, tq, tk, tv, idx, ks, o3, None, ws_t)
    o3h = garbage_like(dq.shape)
    T.tsa_attend_gathered(p_h, dq, dk, dv, idx, ks, o3h, None, ws_h)
    assert torch.equal(head_major(o3).view(torch.int16), o3h.view(torch.int16))
    # dense attention on the token-major tensors
    od_h, od_t = garbage_like(dq.shape), garbage_like(tq.shape)
    T.tsa_attend_dense(p_h, dq, dk, dv, od_h, None, ws_h)
    T.tsa_attend_dense(p_t, tq, tk, tv, od_t, None, ws_t)
    assert torch.equal(head_major(od_t).view(torch.int16), od_h.view(torch.int16))
    rows = np.array([0, 1, wl.L // 2, wl.L - 1])
    ref = O.attention_rows(q[0, 1], k[0, 1 // wl.G], v[0, 1 // wl.G], rows, O.default_scale(wl.d))
    got = bf16_to_f64(od_t[0, torch.from_numpy(rows).cuda(), 1])
    assert np.abs(got - ref).max() <= ATOL_OUT
    assert_status_clean(ws_h)
    assert_status_clean(ws_t)


def test_forward_token_major_32k_sampled():
    wl = W.WORKLOADS["c3_L32K_gqa_band"]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    tq, tk, tv = tok_major(dq), tok_major(dk), tok_major(dv)
    del dq, dk, dv
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, layout="blhd")
    o, s, idx, ks = run_forward(wl, p, tq, tk, tv, tq.shape)
    g_s, g_idx, g_ks = s.cpu().numpy(), idx.cpu().numpy(), ks.cpu().numpy()
    _, ks_ref = O.coverage_budget(g_s, wl.tau)
    assert np.array_equal(g_ks, ks_ref)
    assert np.array_equal(g_idx, O.select_topk(g_s, ks_ref))
    rng = np.random.default_rng(9)
    for h in (0, 17, wl.Hq - 1):
        rows = sample_rows(wl.L, rng, n=8)
        ref = O.output_rows(q, k, v, g_idx, g_ks, 0, h, rows)
        got = bf16_to_f64(o[0, torch.from_numpy(rows).cuda(), h])
        assert np.abs(got - ref).max() <= ATOL_OUT, h
    # unselected rows exactly zero (token-major indexing)
    sel = torch.zeros((wl.Hq, wl.L), dtype=torch.bool, device="cuda")
    sel.scatter_(1, idx[0, :, :int(g_ks[0])].long(), True)
    nz = (o[0].view(torch.int16) != 0).any(dim=-1).transpose(0, 1)
    assert not (nz & ~sel).any().item()
