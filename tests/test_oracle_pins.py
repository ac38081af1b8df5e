"""Pins of the CPU oracle against things other than itself.

Each oracle step is checked against at least one of: hand-derived fixtures
(tests/golden), closed forms, pure-Python brute force on tiny inputs, exhaustive
subset enumeration, and an independent library routine (torch fp64
scaled-dot-product attention).  The planted-mistake tests at the end mutate a
copy of an oracle step on the CPU and show that the pins reject it.

Method source: gist.science summary page "Token Sparse Attention: Efficient
Long-Context Inference with Interleaved Token Selection", section 2
"Metodologia" ("Arquitectura Central", "Cobertura Dinamica de Tokens").
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# fixture parsing
# --------------------------------------------------------------------------
def _budget_examples():
    blocks, cur = [], None
    with open(os.path.join(GOLDEN, "budget_select_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = [t.strip() for t in line.split(":", 1)]
            if key == "name":
                cur = {"name": val, "heads": []}
                blocks.append(cur)
            elif key == "head":
                cur["heads"].append([float(t) for t in val.split()])
            elif key == "tau":
                cur["tau"] = float(val)
            elif key in ("T", "k_head"):
                cur[key] = [int(t) for t in val.split()]
            elif key == "k_seq":
                cur[key] = int(val)
            elif key == "idx":
                cur[key] = [[int(t) for t in part.split()] for part in val.split("|")]
    return blocks


def _score_attention_examples():
    vals = {}
    with open(os.path.join(GOLDEN, "score_attention_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            vals[key.strip()] = [float(t) for t in val.split()]
    return vals


# --------------------------------------------------------------------------
# brute-force references (pure Python, written from the definitions)
# --------------------------------------------------------------------------
def brute_scores(q_rows, k_rows, L, w, scale):
    """Column sums of the causal softmax rows of the last w queries."""
    score = [0.0] * L
    for r in range(w):
        i = L - w + r
        xs = [scale * sum(a * b for a, b in zip(q_rows[r], k_rows[j])) for j in range(i + 1)]
        m = max(xs)
        es = [math.exp(x - m) for x in xs]
        z = math.fsum(es)
        for j in range(i + 1):
            score[j] += es[j] / z
    return score


def brute_attention(q, k, v, scale):
    out = []
    for i in range(len(q)):
        xs = [scale * sum(a * b for a, b in zip(q[i], k[j])) for j in range(i + 1)]
        m = max(xs)
        es = [math.exp(x - m) for x in xs]
        z = math.fsum(es)
        out.append([math.fsum(es[j] * v[j][t] for j in range(i + 1)) / z for t in range(len(v[0]))])
    return out


def exact_mass(s):
    """ceil(s * 2^40) with rational arithmetic."""
    return math.ceil(Fraction(float(np.float32(s))) * (2 ** 40))


def brute_prune_count(scores, tau):
    """Largest subset (any subset, exhaustive) whose exact mass is <= T."""
    qv = [exact_mass(s) for s in scores]
    T = math.floor(float(np.float32(tau)) * float(sum(qv)))
    best = 0
    n = len(qv)
    for r in range(n, -1, -1):
        if any(sum(c) <= T for c in itertools.combinations(qv, r)):
            best = r
            break
    return best


def brute_topk(scores, k):
    """j is kept iff fewer than k tokens rank before it (score desc, index asc)."""
    s = [float(np.float32(x)) for x in scores]
    keep = []
    for j in range(len(s)):
        before = sum(1 for i in range(len(s)) if s[i] > s[j] or (s[i] == s[j] and i < j))
        if before < k:
            keep.append(j)
    return keep


# --------------------------------------------------------------------------
# checks shared by the real tests and the planted-mistake tests
# --------------------------------------------------------------------------
def check_score_fixtures(score_head_fn):
    g = _score_attention_examples()
    # S1: uniform logits
    q = np.ones((2, 2))
    k = np.zeros((4, 2))
    _, s64 = score_head_fn(q, k, 4, O.default_scale(2), True)
    np.testing.assert_allclose(s64, g["S1 score"], rtol=0, atol=1e-15)
    # S2: two keys, scale 1
    _, s64 = score_head_fn(np.array([[0.0], [1.0]]), np.array([[0.0], [2.0]]), 2, 1.0, True)
    np.testing.assert_allclose(s64, g["S2 score"], rtol=0, atol=1e-15)
    # S3: single token
    _, s64 = score_head_fn(np.array([[0.3]]), np.array([[0.7]]), 1, 1.0, True)
    np.testing.assert_allclose(s64, g["S3 score"], rtol=0, atol=0)


def check_budget_fixtures(budget_fn, select_fn):
    for ex in _budget_examples():
        scores = np.array([ex["heads"]], dtype=np.float32)        # [1, H, L]
        qv = O.quantise_mass(scores[0])
        T = O.coverage_threshold(qv, ex["tau"])
        assert list(T) == ex["T"], ex["name"]
        k_head, k_seq = budget_fn(scores, ex["tau"])
        assert list(k_head[0]) == ex["k_head"], ex["name"]
        assert int(k_seq[0]) == ex["k_seq"], ex["name"]
        idx = select_fn(scores, k_seq)
        for h, want in enumerate(ex["idx"]):
            assert list(idx[0, h, :ex["k_seq"]]) == want, ex["name"]
            assert (idx[0, h, ex["k_seq"]:] == -1).all()


def check_attention_fixtures(rows_fn):
    g = _score_attention_examples()
    v = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]])
    o = rows_fn(np.zeros((3, 2)), np.zeros((3, 2)), v, np.arange(3), 1.0)
    np.testing.assert_allclose(o.ravel(), g["A1 out"], rtol=0, atol=1e-15)
    o = rows_fn(np.array([[1.0], [1.0]]), np.array([[0.0], [2.0]]), np.array([[1.0], [0.0]]),
                np.arange(2), 1.0)
    np.testing.assert_allclose(o.ravel(), g["A2 out"], rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# proxy scores
# --------------------------------------------------------------------------
def test_scores_fixtures():
    check_score_fixtures(O.proxy_scores_head)


@pytest.mark.parametrize("L,w,d", [(12, 5, 3), (9, 9, 2), (16, 1, 4)])
def test_scores_brute_force(L, w, d):
    rng = np.random.default_rng(L * 100 + w)
    q = rng.standard_normal((w, d)) * 2
    k = rng.standard_normal((L, d)) * 2
    scale = 0.37
    _, s64 = O.proxy_scores_head(q, k, L, scale, True)
    ref = brute_scores(q.tolist(), k.tolist(), L, w, scale)
    np.testing.assert_allclose(s64, ref, rtol=1e-13, atol=1e-15)


def test_scores_uniform_closed_form():
    L, w = 300, 37
    q = np.random.default_rng(1).standard_normal((w, 8))
    k = np.zeros((L, 8))
    _, s64 = O.proxy_scores_head(q, k, L, O.default_scale(8), True)
    ref = [sum(1.0 / (i + 1) for i in range(max(j, L - w), L)) for j in range(L)]
    np.testing.assert_allclose(s64, ref, rtol=1e-13, atol=0)


def test_scores_sum_to_window_and_gqa_mapping():
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(Hq=4, Hkv=2, L=96, w=7, heavy_count=3)
    q, k, _ = W.generate(wl)
    s32, s64 = O.proxy_scores(q, k, wl.w, return_f64=True)
    np.testing.assert_allclose(s64.sum(-1), wl.w, rtol=1e-12)
    assert np.array_equal(s32, s64.astype(np.float32))
    qf, kf = W.bf16_bits_to_f64(q), W.bf16_bits_to_f64(k)
    scale = O.default_scale(wl.d)
    for h in range(wl.Hq):  # head h reads KV head h // G (consecutive grouping)
        ref = brute_scores(qf[0, h, wl.L - wl.w:].tolist(), kf[0, h // 2].tolist(), wl.L, wl.w, scale)
        np.testing.assert_allclose(s64[0, h], ref, rtol=1e-12, atol=1e-300)


# --------------------------------------------------------------------------
# coverage budget and selection
# --------------------------------------------------------------------------
def test_budget_and_select_fixtures():
    check_budget_fixtures(O.coverage_budget, O.select_topk)


@pytest.mark.parametrize("seed", range(12))
def test_budget_matches_subset_enumeration(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(2, 12))
    # a few repeated values and a few exact zeros, like real score vectors
    base = rng.exponential(size=L) * (rng.random(L) > 0.15)
    if seed % 3 == 0:
        base = np.round(base * 2) / 2
    scores = (base / max(base.sum(), 1e-3) * 7).astype(np.float32)
    scores[rng.integers(0, L)] += np.float32(0.5)
    tau = float(rng.choice([0.0, 0.01, 0.05, 0.1, 0.3, 0.5, 0.9]))
    p = O.pruned_count_head(scores, tau)
    assert p == brute_prune_count(scores, tau)


def test_budget_equal_scores_closed_form():
    for L, s, tau in [(1000, 0.0625, 0.05), (4096, 2.0 ** -10, 0.1), (7, 0.5, 0.99)]:
        scores = np.full(L, s, dtype=np.float32)
        q1 = exact_mass(s)
        T = math.floor(float(np.float32(tau)) * float(q1 * L))
        assert O.pruned_count_head(scores, tau) == min(L, T // q1)


def test_budget_invariants_on_workload():
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"]
    q, k, _ = W.generate(wl)
    scores = O.proxy_scores(q, k, wl.w)
    for tau in (0.0, 0.01, 0.05, 0.2):
        k_head, k_seq = O.coverage_budget(scores, tau)
        for h in range(wl.Hq):
            qv = O.quantise_mass(scores[0, h])
            T = int(O.coverage_threshold(qv, tau))
            srt = np.sort(qv)
            p = wl.L - int(k_head[0, h])
            assert int(srt[:p].sum()) <= T                   # pruned mass within tau
            if p < wl.L:
                assert int(srt[:p + 1].sum()) > T            # one more would exceed
        assert k_seq[0] == k_head[0].max()
        if tau == 0.0:
            assert (k_head == wl.L).all()
    # a larger threshold never keeps more tokens
    ks = [O.coverage_budget(scores, t)[0] for t in (0.0, 0.01, 0.05, 0.2, 0.6)]
    for a, b in zip(ks, ks[1:]):
        assert (b <= a).all()


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_rank_definition(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(5, 60))
    scores = rng.choice(np.array([0.0, 0.25, 0.5, 1.0, 3.0], dtype=np.float32), size=L)
    for k in sorted({1, L // 3, L // 2, L}):
        got = O.select_head(scores, max(k, 1))
        assert list(got) == brute_topk(scores, max(k, 1))
        assert np.all(np.diff(got) > 0)


# --------------------------------------------------------------------------
# gather / scatter
# --------------------------------------------------------------------------
def test_gather_scatter_placement():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, L, d = 2, 4, 2, 50, 8
    q = rng.integers(0, 2 ** 16, size=(B, Hq, L, d), dtype=np.uint16)
    k = rng.integers(0, 2 ** 16, size=(B, Hkv, L, d), dtype=np.uint16)
    v = rng.integers(0, 2 ** 16, size=(B, Hkv, L, d), dtype=np.uint16)
    k_seq = np.array([17, 50], dtype=np.int32)
    idx = np.full((B, Hq, L), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            idx[b, h, :k_seq[b]] = np.sort(rng.choice(L, size=k_seq[b], replace=False))
    qc, kc, vc = O.gather_qkv(q, k, v, idx, k_seq)
    for b in range(B):
        for h in range(Hq):
            for i in range(L):
                if i < k_seq[b]:
                    j = idx[b, h, i]
                    assert (qc[b, h, i] == q[b, h, j]).all()
                    assert (kc[b, h, i] == k[b, h // 2, j]).all()
                    assert (vc[b, h, i] == v[b, h // 2, j]).all()
                else:
                    assert (qc[b, h, i] == 0).all() and (kc[b, h, i] == 0).all()
    oc = rng.standard_normal((B, Hq, L, d))
    o = O.scatter(oc, idx, k_seq, L)
    for b in range(B):
        for h in range(Hq):
            sel = set(idx[b, h, :k_seq[b]].tolist())
            for r in range(L):
                if r in sel:
                    i = int(np.where(idx[b, h] == r)[0][0])
                    assert (o[b, h, r] == oc[b, h, i]).all()
                else:
                    assert (o[b, h, r] == 0).all() and not np.signbit(o[b, h, r]).any()


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def test_attention_fixtures():
    check_attention_fixtures(O.attention_rows)


def test_attention_brute_force():
    rng = np.random.default_rng(5)
    L, d = 9, 3
    q, k, v = (rng.standard_normal((L, d)) * 1.5 for _ in range(3))
    got = O.attention_rows(q, k, v, np.arange(L), 0.8)
    np.testing.assert_allclose(got, brute_attention(q.tolist(), k.tolist(), v.tolist(), 0.8),
                               rtol=1e-13, atol=1e-14)
    # rows evaluated out of order / in chunks agree (BLAS blocking may differ)
    perm = rng.permutation(L)
    np.testing.assert_allclose(O.attention_rows(q, k, v, perm, 0.8, chunk=2), got[perm],
                               rtol=1e-13, atol=1e-14)


def test_dense_attention_matches_torch_sdpa_fp64():
    import torch
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(Hq=4, Hkv=2, L=80, d=16)
    q, k, v = W.generate(wl)
    got = O.dense_causal_attention(q, k, v)
    tq, tk, tv = (torch.from_numpy(W.bf16_bits_to_f64(x)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=True, scale=O.default_scale(wl.d), enable_gqa=True).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_single_token_and_tau_zero_identity():
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(L=200)
    q, k, v = W.generate(wl)
    # k = 1: the single compressed row attends only itself -> its V row
    qc, kc, vc = q[0, 0, :1], k[0, 0, :1], v[0, 0, :1]
    o = O.attention_rows(qc, kc, vc, [0], 0.125)
    assert np.array_equal(o[0], W.bf16_bits_to_f64(vc[0]))
    # tau = 0 keeps every token; the path then equals dense causal attention
    res = O.forward(q, k, v, wl.w, 0.0)
    assert (res["k_seq"] == wl.L).all()
    assert (res["idx"] == np.arange(wl.L)[None, None, :]).all()
    assert np.array_equal(res["o"], O.dense_causal_attention(q, k, v))


def test_forward_invariants_and_row_sampler():
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(L=300, w=16)
    q, k, v = W.generate(wl)
    res = O.forward(q, k, v, wl.w, 0.1)
    kb = int(res["k_seq"][0])
    assert 1 <= kb < wl.L
    for h in range(wl.Hq):
        s = res["idx"][0, h, :kb]
        assert np.all(np.diff(s) > 0) and (res["idx"][0, h, kb:] == -1).all()
        unsel = np.setdiff1d(np.arange(wl.L), s)
        assert (res["o"][0, h, unsel] == 0).all()
        rows = np.arange(0, wl.L, 7)
        got = O.output_rows(q, k, v, res["idx"], res["k_seq"], 0, h, rows)
        np.testing.assert_allclose(got, res["o"][0, h, rows], rtol=1e-12, atol=1e-13)
        assert (got[~np.isin(rows, s)] == 0).all()


# --------------------------------------------------------------------------
# planted mistakes: each mutated copy of an oracle step must fail a pin
# --------------------------------------------------------------------------
def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_planted_mistakes_are_caught():
    # proxy map without the causal mask
    def no_mask(qw, kh, L, scale, ret):
        x = (np.asarray(qw, float) @ np.asarray(kh, float).T) * scale
        e = np.exp(x - x.max(1, keepdims=True))
        s = (e / e.sum(1, keepdims=True)).sum(0)
        return s.astype(np.float32), s
    assert _fails(check_score_fixtures, no_mask)

    # column sum of unnormalised weights
    def no_norm(qw, kh, L, scale, ret):
        w = qw.shape[0]
        x = (np.asarray(qw, float) @ np.asarray(kh, float).T) * scale
        x = np.where(np.arange(L)[None] <= np.arange(L - w, L)[:, None], x, -np.inf)
        s = np.exp(x - x.max(1, keepdims=True)).sum(0)
        return s.astype(np.float32), s
    assert _fails(check_score_fixtures, no_norm)

    # budget variants: descending order, strict comparison, min over heads
    def budget_with(order_desc=False, strict=False, agg=np.max):
        def fn(scores, tau):
            B, H, L = scores.shape
            kh = np.empty((B, H), np.int32)
            for b in range(B):
                for h in range(H):
                    qv = O.quantise_mass(scores[b, h])
                    T = int(O.coverage_threshold(qv, tau))
                    srt = np.sort(qv)[::-1] if order_desc else np.sort(qv)
                    cum = np.cumsum(srt)
                    kh[b, h] = L - int(np.count_nonzero(cum < T if strict else cum <= T))
            return kh, agg(kh, axis=1).astype(np.int32)
        return fn
    assert _fails(check_budget_fixtures, budget_with(order_desc=True), O.select_topk)
    assert _fails(check_budget_fixtures, budget_with(strict=True), O.select_topk)
    assert _fails(check_budget_fixtures, budget_with(agg=np.min), O.select_topk)

    # ties broken toward the larger index
    def select_bad_ties(scores, k_seq):
        B, H, L = scores.shape
        idx = np.full((B, H, L), -1, np.int32)
        for b in range(B):
            for h in range(H):
                order = np.lexsort((-np.arange(L), -scores[b, h].astype(float)))
                idx[b, h, :k_seq[b]] = np.sort(order[:k_seq[b]])
        return idx
    assert _fails(check_budget_fixtures, O.coverage_budget, select_bad_ties)

    # attention with V and K swapped
    def swapped(q, k, v, rows, scale, chunk=1024):
        return O.attention_rows(q, v, k, rows, scale, chunk)
    assert _fails(check_attention_fixtures, swapped)
