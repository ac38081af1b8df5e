"""GPU parity of every step of the path against the CPU oracle, through the
C ABI, at sizes the oracle finishes in seconds (several 128-row tiles, ragged
tails, MHA and GQA, d = 64 and 128, window blocks > 128 rows).

Tolerances (fixed by the method's accuracy targets):
  scores      |gpu - oracle| <= 1e-5 |oracle| + 1e-30 (oracle in fp64)
  budget, selection, gather, scatter: bit-exact (fed the same inputs)
  attention   max |gpu - oracle| <= 2e-2 (bf16 in/out, fp32 accumulation)
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, from_dev_bf16, garbage_like, inputs, scores_close, to_dev_bf16

pytestmark = pytest.mark.gpu

ATOL_OUT = 2e-2

BASE = W.WORKLOADS["c1_L1K_mha_d64"]
SHAPES = {
    "c1_mha_d64_L1024": BASE,
    "gqa_d128_L1000": BASE.with_(Hq=4, Hkv=2, L=1000, d=128, w=48, tau=0.1, heavy_count=0,
                                 heavy_frac_lo=0.01, heavy_frac_hi=0.01, heavy_scale=3.0, sink=False, seed=11),
    "gqa_d128_B2_L777_w130": BASE.with_(B=2, Hq=6, Hkv=2, L=777, d=128, w=130, tau=0.05, heavy_count=5,
                                        heavy_scale=3.0, seed=12),
    "mha_d128_L129": BASE.with_(Hq=2, Hkv=2, L=129, d=128, w=7, tau=0.3, heavy_count=2, seed=13),
    "gqa_d64_L2500": BASE.with_(Hq=8, Hkv=2, L=2500, d=64, w=64, tau=0.2, heavy_count=0, heavy_frac_lo=0.001,
                                heavy_frac_hi=0.02, heavy_scale=3.0, seed=14, band_half=16, band_a=0.5),
    "single_token": BASE.with_(Hq=2, Hkv=1, L=1, d=64, w=1, tau=0.05, heavy_count=0, sink=False, seed=15),
}


def P(wl, tau=None):
    return T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau if tau is None else tau)


def dev_i32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def assert_status_clean(ws):
    st, flags = T.get_device_status(ws)
    assert st == 0 and flags == 0, (st, flags)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    T.load()


@pytest.mark.parametrize("name", list(SHAPES))
def test_score_parity(name):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = P(wl)
    ws = T.new_workspace(p, full=False)
    scores = torch.full((wl.B, wl.Hq, wl.L), float("nan"), device="cuda")
    T.tsa_score(p, dq, dk, scores, ws)
    _, ref64 = O.proxy_scores(q, k, wl.w, return_f64=True)
    worst = scores_close(scores.cpu().numpy(), ref64)
    assert worst <= 1.0, f"score error {worst:.3f} x tolerance"
    assert_status_clean(ws)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("tau", [0.0, 0.01, 0.05, 0.3, 0.9])
def test_budget_select_bit_exact(name, tau):
    wl = SHAPES[name]
    q, k, _ = W.generate(wl)
    s32 = O.proxy_scores(q, k, wl.w)          # the oracle's fp32 scores feed both sides
    k_head, k_seq = O.coverage_budget(s32, tau)
    idx = O.select_topk(s32, k_seq)
    p = P(wl, tau)
    ws = T.new_workspace(p, full=False)
    ds = torch.from_numpy(s32).cuda()
    g_kh = torch.full((wl.B, wl.Hq), -7, dtype=torch.int32, device="cuda")
    g_ks = torch.full((wl.B,), -7, dtype=torch.int32, device="cuda")
    g_idx = torch.full((wl.B, wl.Hq, wl.L), -7, dtype=torch.int32, device="cuda")
    T.tsa_budget(p, ds, g_kh, g_ks, ws)
    T.tsa_select(p, ds, g_ks, g_idx, ws)
    assert np.array_equal(g_kh.cpu().numpy(), k_head)
    assert np.array_equal(g_ks.cpu().numpy(), k_seq)
    assert np.array_equal(g_idx.cpu().numpy(), idx)
    assert_status_clean(ws)


def test_budget_select_golden_fixtures():
    import test_oracle_pins as pins
    for ex in pins._budget_examples():
        s = np.array([ex["heads"]], dtype=np.float32)
        H, L = s.shape[1], s.shape[2]
        p = T.params(1, H, 1, L, 64, 1, ex["tau"])
        ws = T.new_workspace(p, full=False)
        kh = torch.empty((1, H), dtype=torch.int32, device="cuda")
        ks = torch.empty((1,), dtype=torch.int32, device="cuda")
        ix = torch.empty((1, H, L), dtype=torch.int32, device="cuda")
        ds = torch.from_numpy(s).cuda()
        T.tsa_budget(p, ds, kh, ks, ws)
        T.tsa_select(p, ds, ks, ix, ws)
        assert list(kh.cpu().numpy()[0]) == ex["k_head"], ex["name"]
        assert int(ks.cpu()[0]) == ex["k_seq"], ex["name"]
        for h, want in enumerate(ex["idx"]):
            assert list(ix.cpu().numpy()[0, h, :ex["k_seq"]]) == want, ex["name"]


@pytest.mark.parametrize("seed", range(4))
def test_select_many_ties_and_zero_scores(seed):
    rng = np.random.default_rng(seed)
    B, H, L = 2, 3, 5000 + 37 * seed
    s = rng.choice(np.array([0.0, 1e-30, 2.0 ** -20, 0.5, 0.5, 3.0], dtype=np.float32), size=(B, H, L))
    s[:, :, 7] = 100.0
    for tau in (0.0, 0.05, 0.5):
        k_head, k_seq = O.coverage_budget(s, tau)
        idx = O.select_topk(s, k_seq)
        p = T.params(B, H, 1, L, 64, 1, tau)
        ws = T.new_workspace(p, full=False)
        ds = torch.from_numpy(s).cuda()
        kh = torch.empty((B, H), dtype=torch.int32, device="cuda")
        ks = torch.empty((B,), dtype=torch.int32, device="cuda")
        ix = torch.empty((B, H, L), dtype=torch.int32, device="cuda")
        T.tsa_budget(p, ds, kh, ks, ws)
        T.tsa_select(p, ds, ks, ix, ws)
        assert np.array_equal(kh.cpu().numpy(), k_head)
        assert np.array_equal(ks.cpu().numpy(), k_seq)
        assert np.array_equal(ix.cpu().numpy(), idx)


def test_budget_flags_nonfinite_scores():
    s = np.full((1, 2, 300), 0.01, dtype=np.float32)
    s[0, 1, 17] = np.nan
    p = T.params(1, 2, 1, 300, 64, 1, 0.05)
    ws = T.new_workspace(p, full=False)
    ks = torch.empty((1,), dtype=torch.int32, device="cuda")
    T.tsa_budget(p, torch.from_numpy(s).cuda(), None, ks, ws)
    st, flags = T.get_device_status(ws)
    assert st == 5 and flags & T.DEVFLAG_NONFINITE
    T.reset_device_status(ws)
    assert_status_clean(ws)


@pytest.mark.parametrize("name", ["c1_mha_d64_L1024", "gqa_d128_B2_L777_w130", "gqa_d64_L2500"])
def test_gather_scatter_bit_exact(name):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    rng = np.random.default_rng(5)
    k_seq = np.array([max(1, int(wl.L * f)) for f in rng.uniform(0.3, 1.0, wl.B)], dtype=np.int32)
    idx = np.full((wl.B, wl.Hq, wl.L), -1, dtype=np.int32)
    for b in range(wl.B):
        for h in range(wl.Hq):
            idx[b, h, :k_seq[b]] = np.sort(rng.choice(wl.L, size=k_seq[b], replace=False))
    p = P(wl)
    ref_q, ref_k, ref_v = O.gather_qkv(q, k, v, idx, k_seq)
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    qc, kc, vc = garbage_like(shape), garbage_like(shape), garbage_like(shape)
    dix, dks = dev_i32(idx), dev_i32(k_seq)
    T.tsa_gather_qkv(p, dq, dk, dv, dix, dks, qc, kc, vc)
    for g, r in ((qc, ref_q), (kc, ref_k), (vc, ref_v)):
        gb = from_dev_bf16(g)
        for b in range(wl.B):
            assert np.array_equal(gb[b, :, :k_seq[b]], r[b, :, :k_seq[b]])
            assert (gb[b, :, k_seq[b]:] == 0x7FC1).all()        # rows >= k_b untouched
    # scatter an arbitrary compressed output back
    oc_bits = W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    ref_o = O.scatter(oc_bits, idx, k_seq, wl.L)
    o = garbage_like(shape)
    T.tsa_scatter(p, to_dev_bf16(oc_bits), dix, dks, o)
    assert np.array_equal(from_dev_bf16(o), ref_o)


def _compressed_case(wl, tau):
    (q, k, v), _ = inputs(wl)
    s32 = O.proxy_scores(q, k, wl.w)
    _, k_seq = O.coverage_budget(s32, tau)
    idx = O.select_topk(s32, k_seq)
    qc, kc, vc = O.gather_qkv(q, k, v, idx, k_seq)
    return (q, k, v), k_seq, idx, (qc, kc, vc)


@pytest.mark.parametrize("name", [n for n in SHAPES])
@pytest.mark.parametrize("tau", [0.05, 0.6])
def test_attend_parity(name, tau):
    wl = SHAPES[name]
    _, k_seq, idx, (qc, kc, vc) = _compressed_case(wl, tau)
    p = P(wl, tau)
    ws = T.new_workspace(p, full=False)
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    # rows >= k_b hold NaN garbage: the kernel must not let them leak
    dq, dk, dv = garbage_like(shape), garbage_like(shape), garbage_like(shape)
    for dst, src in ((dq, qc), (dk, kc), (dv, vc)):
        for b in range(wl.B):
            dst[b, :, :k_seq[b]] = to_dev_bf16(src[b, :, :k_seq[b]])
    oc = garbage_like(shape)
    lse = torch.full((wl.B, wl.Hq, wl.L), float("nan"), device="cuda")
    T.tsa_attend(p, dq, dk, dv, dev_i32(k_seq), oc, lse, ws)
    ref = O.compressed_attention(qc, kc, vc, k_seq)
    got = bf16_to_f64(oc)
    scale = O.default_scale(wl.d)
    for b in range(wl.B):
        kb = int(k_seq[b])
        err = np.abs(got[b, :, :kb] - ref[b, :, :kb]).max()
        assert err <= ATOL_OUT, f"b={b} max err {err}"
        assert (from_dev_bf16(oc)[b, :, kb:] == 0x7FC1).all()
        # log-sum-exp of the first and last valid rows, from the definition
        for h in range(wl.Hq):
            for i in (0, kb - 1):
                x = (W.bf16_bits_to_f64(qc[b, h, i]) @ W.bf16_bits_to_f64(kc[b, h, :i + 1]).T) * scale
                want = x.max() + np.log(np.exp(x - x.max()).sum())
                assert abs(float(lse[b, h, i]) - want) < 1e-3
    assert_status_clean(ws)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("tau", [0.05, 0.6])
def test_attend_gathered_parity(name, tau):
    """Gather, attention and scatter fused in one kernel (rows loaded by index,
    outputs written in place, every other row zero) against the oracle."""
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    s32 = O.proxy_scores(q, k, wl.w)
    _, k_seq = O.coverage_budget(s32, tau)
    idx = O.select_topk(s32, k_seq)
    p = P(wl, tau)
    ws = T.new_workspace(p, full=False)
    o = garbage_like(dq.shape)
    lse = torch.full((wl.B, wl.Hq, wl.L), float("nan"), device="cuda")
    T.tsa_attend_gathered(p, dq, dk, dv, dev_i32(idx), dev_i32(k_seq), o, lse, ws)
    qc, kc, vc = O.gather_qkv(q, k, v, idx, k_seq)
    oc = O.compressed_attention(qc, kc, vc, k_seq)
    ref = O.scatter(oc, idx, k_seq, wl.L)
    got = bf16_to_f64(o)
    assert np.abs(got - ref).max() <= ATOL_OUT
    bits = from_dev_bf16(o)
    scale = O.default_scale(wl.d)
    for b in range(wl.B):
        kb = int(k_seq[b])
        for h in range(wl.Hq):
            unsel = np.setdiff1d(np.arange(wl.L), idx[b, h, :kb])
            assert (bits[b, h, unsel] == 0).all()
            i = kb - 1     # the last compressed row's log-sum-exp
            x = (W.bf16_bits_to_f64(qc[b, h, i]) @ W.bf16_bits_to_f64(kc[b, h, :i + 1]).T) * scale
            assert abs(float(lse[b, h, i]) - (x.max() + np.log(np.exp(x - x.max()).sum()))) < 1e-3
    assert_status_clean(ws)


@pytest.mark.parametrize("name", list(SHAPES))
def test_attend_scatter_parity(name):
    """The path tsa_forward runs: Q, K, V gathered once, then attention with
    the scatter in its epilogue (outputs written in place, the rest zero)."""
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    s32 = O.proxy_scores(q, k, wl.w)
    _, k_seq = O.coverage_budget(s32, wl.tau)
    idx = O.select_topk(s32, k_seq)
    p = P(wl)
    ws = T.new_workspace(p, full=False)
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    qc_d, kc, vc, o = (garbage_like(shape) for _ in range(4))
    dix, dks = dev_i32(idx), dev_i32(k_seq)
    T.tsa_gather_qkv(p, dq, dk, dv, dix, dks, None, kc, vc, ws)      # K/V-only form
    T.tsa_gather_qkv(p, dq, dk, dv, dix, dks, qc_d, kc, vc, ws)
    T.tsa_attend_scatter(p, qc_d, kc, vc, dix, dks, o, None, ws)
    qc, kc_ref, vc_ref = O.gather_qkv(q, k, v, idx, k_seq)
    for b in range(wl.B):      # the K/V-only gather is bit-exact
        kb = int(k_seq[b])
        assert np.array_equal(from_dev_bf16(kc)[b, :, :kb], kc_ref[b, :, :kb])
        assert np.array_equal(from_dev_bf16(vc)[b, :, :kb], vc_ref[b, :, :kb])
    ref = O.scatter(O.compressed_attention(qc, kc_ref, vc_ref, k_seq), idx, k_seq, wl.L)
    assert np.abs(bf16_to_f64(o) - ref).max() <= ATOL_OUT
    bits = from_dev_bf16(o)
    for b in range(wl.B):
        for h in range(wl.Hq):
            unsel = np.setdiff1d(np.arange(wl.L), idx[b, h, :k_seq[b]])
            assert (bits[b, h, unsel] == 0).all()
    assert_status_clean(ws)


def test_attend_gathered_flags_bad_index():
    wl = SHAPES["gqa_d128_L1000"]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    k_seq = np.array([300], dtype=np.int32)
    idx = np.full((1, wl.Hq, wl.L), -1, dtype=np.int32)
    for h in range(wl.Hq):
        idx[0, h, :300] = np.arange(0, 900, 3)
    idx[0, 1, 299] = wl.L + 5           # out of range: skipped and flagged, never written
    p = P(wl)
    ws = T.new_workspace(p, full=False)
    o = garbage_like(dq.shape)
    T.tsa_attend_gathered(p, dq, dk, dv, dev_i32(idx), dev_i32(k_seq), o, None, ws)
    st, flags = T.get_device_status(ws)
    assert flags & T.DEVFLAG_BAD_INDEX
    qc, kc, vc = O.gather_qkv(q, k, v, np.where(idx >= 0, np.minimum(idx, wl.L - 1), -1), k_seq)
    ref = O.compressed_attention(qc, kc, vc, k_seq)
    got = bf16_to_f64(o)
    for h in (0, 2, 3):                  # heads with valid indices are unaffected
        assert np.abs(got[0, h, idx[0, h, :300]] - ref[0, h, :300]).max() <= ATOL_OUT
    T.reset_device_status(ws)


@pytest.mark.parametrize("name", ["c1_mha_d64_L1024", "gqa_d128_L1000", "gqa_d128_B2_L777_w130", "mha_d128_L129"])
def test_attend_dense_parity(name):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = P(wl)
    ws = T.new_workspace(p, full=False)
    o = garbage_like(dq.shape)
    T.tsa_attend_dense(p, dq, dk, dv, o, None, ws)
    ref = O.dense_causal_attention(q, k, v)
    err = np.abs(bf16_to_f64(o) - ref).max()
    assert err <= ATOL_OUT, err
    assert_status_clean(ws)


def near_tie_ok(s_oracle_head, got, want, rel=2e-5):
    """Tokens on which two selections differ must sit at the threshold."""
    diff = np.setxor1d(got, want)
    if diff.size == 0:
        return True
    kth = np.sort(s_oracle_head.astype(np.float64))[::-1][max(len(want), 1) - 1]
    return bool(np.all(np.abs(s_oracle_head[diff] - kth) <= rel * max(kth, 1e-30)))


@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_end_to_end(name):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = P(wl)
    ws = T.new_workspace(p, full=True)
    o = garbage_like(dq.shape)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    k_seq = torch.empty((wl.B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, k_seq)
    g_s, g_idx, g_ks = scores.cpu().numpy(), idx.cpu().numpy(), k_seq.cpu().numpy()
    # (a) scores within tolerance of the fp64 definition
    o_s32, o_s64 = O.proxy_scores(q, k, wl.w, return_f64=True)
    assert scores_close(g_s, o_s64) <= 1.0
    # (b) budget and selection are exactly the oracle's on the GPU's own scores
    _, ks_on_g = O.coverage_budget(g_s, wl.tau)
    assert np.array_equal(g_ks, ks_on_g)
    assert np.array_equal(g_idx, O.select_topk(g_s, ks_on_g))
    # (c) output = oracle attention over the GPU's selection; zeros elsewhere
    qc, kc, vc = O.gather_qkv(q, k, v, g_idx, g_ks)
    ref = O.scatter(O.compressed_attention(qc, kc, vc, g_ks), g_idx, g_ks, wl.L)
    got = bf16_to_f64(o)
    assert np.abs(got - ref).max() <= ATOL_OUT
    for b in range(wl.B):
        for h in range(wl.Hq):
            unsel = np.setdiff1d(np.arange(wl.L), g_idx[b, h, :g_ks[b]])
            assert (from_dev_bf16(o)[b, h, unsel] == 0).all()
    # (d) against the oracle's own path: identical, or differing only at ties
    _, o_ks = O.coverage_budget(o_s32, wl.tau)
    o_idx = O.select_topk(o_s32, o_ks)
    for b in range(wl.B):
        assert abs(int(o_ks[b]) - int(g_ks[b])) <= 1
        for h in range(wl.Hq):
            assert near_tie_ok(o_s64[b, h], g_idx[b, h, :g_ks[b]], o_idx[b, h, :o_ks[b]])
    assert_status_clean(ws)
