"""Pins of the oracle's budget modes and forced keeps (CPU only).

The budget modes ("max", "mean", "per_head") and keep_recent are readings of
the gist.science summary page "Token Sparse Attention: Efficient Long-Context
Inference with Interleaved Token Selection", section 2, "Cobertura Dinamica de
Tokens", which calls the budget global but does not say how the heads'
coverage counts combine.  They are pinned here by hand-derived fixtures
(tests/golden/budget_modes_examples.txt), a brute-force exchange definition
of the forced selection, coverage invariants per head, and an independent
library (torch fp64 scaled-dot-product attention) for the per-head path.
"""
import itertools
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _mode_examples():
    blocks, cur = [], None
    with open(os.path.join(GOLDEN, "budget_modes_examples.txt")) as f:
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
            elif key == "mode":
                cur["mode"] = val
            elif key in ("keep_recent", "k_seq"):
                cur[key] = int(val)
            elif key in ("k_head", "kept"):
                cur[key] = [int(t) for t in val.split()]
            elif key == "idx":
                cur[key] = [[int(t) for t in part.split()] for part in val.split("|")]
    return blocks


def check_mode_fixtures(budget_fn, kept_fn, select_fn):
    ex = _mode_examples()
    assert len(ex) >= 9
    for e in ex:
        scores = np.array([e["heads"]], dtype=np.float32)
        k_head, k_seq = budget_fn(scores, e["tau"], e["mode"], e["keep_recent"])
        assert list(k_head[0]) == e["k_head"], e["name"]
        assert int(k_seq[0]) == e["k_seq"], e["name"]
        kept = kept_fn(k_head, k_seq, e["mode"])
        assert list(kept[0]) == e["kept"], e["name"]
        idx = select_fn(scores, kept, e["keep_recent"])
        for h, want in enumerate(e["idx"]):
            n = e["kept"][h]
            assert list(idx[0, h, :n]) == want, (e["name"], h)
            assert (idx[0, h, n:] == -1).all()


def test_budget_mode_fixtures():
    check_mode_fixtures(O.coverage_budget, O.kept_counts, O.select_topk)


def _valid_forced_selection(scores, S, r):
    """Exchange definition: S holds every forced token, and each unforced
    member beats each non-member (higher score, or equal score and smaller
    index)."""
    L = len(scores)
    forced = set(range(L - r, L))
    if not forced <= S:
        return False
    for i in S - forced:
        for j in set(range(L)) - S:
            if not (scores[i] > scores[j] or (scores[i] == scores[j] and i < j)):
                return False
    return True


@pytest.mark.parametrize("seed", range(10))
def test_forced_selection_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    L = int(rng.integers(2, 9))
    scores = rng.choice(np.array([0.0, 0.125, 0.5, 1.0, 2.0], dtype=np.float32), size=L)
    for r in range(0, L + 1):
        for k in range(max(r, 1), L + 1):
            valid = [set(c) for c in itertools.combinations(range(L), k)
                     if _valid_forced_selection(scores, set(c), r)]
            assert len(valid) == 1
            got = O.select_head(scores, k, r)
            assert set(got.tolist()) == valid[0]
            assert np.all(np.diff(got) > 0)


def test_per_head_and_mean_invariants_on_workload():
    import workloads as W
    wl = W.WORKLOADS["c1_L1K_mha_d64"]
    q, k, _ = W.generate(wl)
    scores = O.proxy_scores(q, k, wl.w)
    for tau in (0.01, 0.05, 0.2):
        kh_max, ks_max = O.coverage_budget(scores, tau, "max")
        kh_ph, ks_ph = O.coverage_budget(scores, tau, "per_head")
        kh_mean, ks_mean = O.coverage_budget(scores, tau, "mean")
        # the per-head counts do not depend on the mode
        assert (kh_max == kh_ph).all() and (kh_max == kh_mean).all()
        kept = O.kept_counts(kh_ph, ks_ph, "per_head")
        for h in range(wl.Hq):
            qv = O.quantise_mass(scores[0, h])
            T = int(O.coverage_threshold(qv, tau))
            srt = np.sort(qv)
            p = wl.L - int(kept[0, h])
            assert int(srt[:p].sum()) <= T                 # own pruned mass within tau
            if p < wl.L:
                assert int(srt[:p + 1].sum()) > T          # one more would exceed
        # the mean lies between the smallest and the largest head
        assert kh_mean[0].min() <= ks_mean[0] <= ks_max[0]
        # forced keeps never lower a count and leave counts >= r unchanged
        r = 300
        kh_r, _ = O.coverage_budget(scores, tau, "per_head", keep_recent=r)
        assert (kh_r == np.maximum(kh_ph, r)).all()


def test_per_head_forward_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(7)
    from workloads import f32_to_bf16_bits, bf16_bits_to_f64
    B, Hq, Hkv, L, d, w = 2, 4, 2, 48, 64, 8
    mk = lambda *s: f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
    q, k, v = mk(B, Hq, L, d), mk(B, Hkv, L, d), mk(B, Hkv, L, d)
    k[:, :, ::5] = f32_to_bf16_bits((bf16_bits_to_f64(k[:, :, ::5]) * 3.0).astype(np.float32))   # uneven importance
    G = Hq // Hkv
    for mode, r in (("per_head", 0), ("per_head", 5), ("mean", 3)):
        res = O.forward(q, k, v, w, 0.3, mode=mode, keep_recent=r)
        kept = res["kept"]
        if mode == "per_head":
            assert (kept == res["k_head"]).all()
            assert len(set(kept.ravel().tolist())) > 1      # heads really differ
        for b in range(B):
            for h in range(Hq):
                n = int(kept[b, h])
                S = res["idx"][b, h, :n].astype(np.int64)
                assert (res["idx"][b, h, n:] == -1).all()
                assert set(range(L - r, L)) <= set(S.tolist())
                qt = torch.from_numpy(bf16_bits_to_f64(q[b, h][S]))[None, None]
                kt = torch.from_numpy(bf16_bits_to_f64(k[b, h // G][S]))[None, None]
                vt = torch.from_numpy(bf16_bits_to_f64(v[b, h // G][S]))[None, None]
                ref = torch.nn.functional.scaled_dot_product_attention(
                    qt, kt, vt, is_causal=True, scale=O.default_scale(d))[0, 0].numpy()
                got = res["o"][b, h]
                assert np.abs(got[S] - ref).max() < 1e-12
                rest = np.setdiff1d(np.arange(L), S)
                assert (got[rest] == 0).all()


def _fails(check, *fns):
    try:
        check(*fns)
    except AssertionError:
        return True
    return False


def test_planted_mistakes_are_caught():
    # mean rounded down instead of up
    def mean_floor(scores, tau, mode="max", keep_recent=0):
        kh, ks = O.coverage_budget(scores, tau, mode, keep_recent)
        if mode == "mean":
            ks = (kh.astype(np.int64).sum(axis=1) // kh.shape[1]).astype(np.int32)
        return kh, ks
    assert _fails(check_mode_fixtures, mean_floor, O.kept_counts, O.select_topk)

    # forced keeps not raising the counts
    def no_raise(scores, tau, mode="max", keep_recent=0):
        return O.coverage_budget(scores, tau, mode, 0)
    assert _fails(check_mode_fixtures, no_raise, O.kept_counts, O.select_topk)

    # forced tokens ranked last instead of first
    def forced_last(scores, kept, keep_recent=0):
        B, H, L = scores.shape
        idx = np.full((B, H, L), -1, np.int32)
        for b in range(B):
            for h in range(H):
                n = int(kept[b, h])
                forced = np.arange(L) >= L - keep_recent
                order = np.lexsort((np.arange(L), -scores[b, h].astype(float), forced))
                idx[b, h, :n] = np.sort(order[:n])
        return idx
    assert _fails(check_mode_fixtures, O.coverage_budget, O.kept_counts, forced_last)

    # per-head mode falling back to the shared budget
    def shared_always(k_head, k_seq, mode="max"):
        return O.kept_counts(k_head, k_seq, "max")
    assert _fails(check_mode_fixtures, O.coverage_budget, shared_always, O.select_topk)


def test_window_longer_than_sequence_covers_it():
    """A sequence shorter than the window: every query row is a window row,
    so each of the L rows of the proxy map sums to one and the scores sum
    to L; pinned against a pure-Python brute force of the definition."""
    import math
    rng = np.random.default_rng(11)
    from workloads import f32_to_bf16_bits, bf16_bits_to_f64
    L, d = 5, 8
    q = f32_to_bf16_bits(rng.standard_normal((1, 1, L, d)).astype(np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((1, 1, L, d)).astype(np.float32))
    s32, s64 = O.proxy_scores(q, k, 9, return_f64=True)
    assert abs(s64[0, 0].sum() - L) < 1e-12
    qf, kf, sc = bf16_bits_to_f64(q)[0, 0], bf16_bits_to_f64(k)[0, 0], O.default_scale(d)
    brute = [0.0] * L
    for i in range(L):
        xs = [sum(qf[i, t] * kf[j, t] for t in range(d)) * sc for j in range(i + 1)]
        m = max(xs)
        z = sum(math.exp(x - m) for x in xs)
        for j in range(i + 1):
            brute[j] += math.exp(xs[j] - m) / z
    assert np.allclose(s64[0, 0], brute, rtol=1e-12, atol=1e-14)


def test_varlen_equal_lengths_matches_batched_forward():
    """Packed sequences of equal length give exactly the batched result."""
    rng = np.random.default_rng(12)
    from workloads import f32_to_bf16_bits
    B, Hq, Hkv, L, d = 3, 4, 2, 40, 64
    mk = lambda *s: f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
    q, k, v = mk(B, Hq, L, d), mk(B, Hkv, L, d), mk(B, Hkv, L, d)
    ref = O.forward(q, k, v, 8, 0.2, mode="per_head", keep_recent=3)
    pk = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(B * L, x.shape[1], d))
    res = O.forward_varlen(pk(q), pk(k), pk(v), [0, L, 2 * L, 3 * L], 8, 0.2, mode="per_head", keep_recent=3)
    for b in range(B):
        assert np.array_equal(res[b]["idx"][0], ref["idx"][b])
        assert np.array_equal(res[b]["kept"][0], ref["kept"][b])
        assert np.array_equal(res[b]["o"][0], ref["o"][b])
    assert np.array_equal(res[0]["o_packed"], ref["o"].transpose(0, 2, 1, 3).reshape(B * L, Hq, d))


def test_varlen_sequences_are_independent():
    """Changing one sequence's tokens leaves every other sequence's result
    unchanged, and the packed output is zero outside the selections."""
    rng = np.random.default_rng(13)
    from workloads import f32_to_bf16_bits
    Hq, Hkv, d = 2, 1, 64
    cu = [0, 17, 17, 60, 61]
    T = cu[-1]
    mk = lambda *s: f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
    q, k, v = mk(T, Hq, d), mk(T, Hkv, d), mk(T, Hkv, d)
    a = O.forward_varlen(q, k, v, cu, 8, 0.1)
    q2 = q.copy()
    q2[17:60] = mk(43, Hq, d)
    b = O.forward_varlen(q2, k, v, cu, 8, 0.1)
    for s in (0, 1, 3):
        assert np.array_equal(a[s]["o"], b[s]["o"])
    assert a[1]["o"].shape[2] == 0                      # an empty sequence
    o = a[0]["o_packed"]
    for s in range(len(cu) - 1):
        n = int(a[s]["k_seq"][0])
        for h in range(Hq):
            sel = cu[s] + a[s]["idx"][0, h, :n]
            rest = np.setdiff1d(np.arange(cu[s], cu[s + 1]), sel)
            assert (o[rest, h] == 0).all()


# --------------------------------------------------------------------------
# block-sparse composition over the compressed sequence
# --------------------------------------------------------------------------
def _rand_bf16(rng, *shape):
    from workloads import f32_to_bf16_bits
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def test_block_mask_all_ones_is_plain_attention():
    rng = np.random.default_rng(21)
    B, H, L, d = 1, 2, 300, 64
    q, k, v = (_rand_bf16(rng, B, H, L, d) for _ in range(3))
    nb = (L + 127) // 128
    kept = np.array([L, 260]).reshape(1, 2)
    ref = O.compressed_attention(q, k, v, kept)
    got = O.compressed_attention(q, k, v, kept, block_mask=np.ones((B, H, nb, nb), np.uint8))
    assert np.array_equal(ref, got)


def test_block_diagonal_mask_is_local_attention_torch():
    """Only the diagonal blocks: every 128-row block attends causally within
    itself, checked block by block against torch fp64 SDPA."""
    rng = np.random.default_rng(22)
    from workloads import bf16_bits_to_f64
    L, d = 333, 64
    q, k, v = (_rand_bf16(rng, 1, 1, L, d) for _ in range(3))
    nb = (L + 127) // 128
    got = O.compressed_attention(q, k, v, np.array([L]), block_mask=np.zeros((1, 1, nb, nb), np.uint8))
    for s in range(0, L, 128):
        e = min(L, s + 128)
        t = lambda x: torch.from_numpy(bf16_bits_to_f64(x[0, 0, s:e]))[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True,
                                                               scale=O.default_scale(d))[0, 0].numpy()
        assert np.abs(got[0, 0, s:e] - ref).max() < 1e-12


def test_block_mask_brute_force():
    """A random mask against a pure-Python loop over the definition."""
    import math
    rng = np.random.default_rng(23)
    from workloads import bf16_bits_to_f64
    L, d = 290, 8
    q, k, v = (_rand_bf16(rng, 1, 1, L, d) for _ in range(3))
    nb = (L + 127) // 128
    bm = (rng.random((1, 1, nb, nb)) < 0.5).astype(np.uint8)
    got = O.compressed_attention(q, k, v, np.array([L]), block_mask=bm)
    qf, kf, vf = (bf16_bits_to_f64(x)[0, 0] for x in (q, k, v))
    sc = O.default_scale(d)
    for i in (0, 127, 128, 200, 255, 256, 289):
        keys = [j for j in range(i + 1) if j // 128 == i // 128 or bm[0, 0, i // 128, j // 128]]
        xs = [sum(qf[i, t] * kf[j, t] for t in range(d)) * sc for j in keys]
        m = max(xs)
        ws = [math.exp(x - m) for x in xs]
        z = sum(ws)
        ref = [sum(ws[a] * vf[j, t] for a, j in enumerate(keys)) / z for t in range(d)]
        assert np.allclose(got[0, 0, i], ref, rtol=1e-12, atol=1e-13)


def test_block_mask_planted_mistake_is_caught():
    """A mask read transposed (key block, query block) fails the brute force."""
    rng = np.random.default_rng(24)
    L, d = 290, 8
    q, k, v = (_rand_bf16(rng, 1, 1, L, d) for _ in range(3))
    bm = np.zeros((1, 1, 3, 3), np.uint8)
    bm[0, 0, 2, 0] = 1                      # block 2 may see block 0
    right = O.compressed_attention(q, k, v, np.array([L]), block_mask=bm)
    wrong = O.compressed_attention(q, k, v, np.array([L]), block_mask=bm.transpose(0, 1, 3, 2).copy())
    assert not np.allclose(right[0, 0, 256:], wrong[0, 0, 256:])
