"""CPU oracle for the Token Sparse Attention prefill path (TEST INFRASTRUCTURE).

This package is test infrastructure, not product code.  Only the test suite,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The CUDA path never calls it, shares no
code with it, and must fail loudly rather than fall back to it.

It is a plain, slow, fp64 restatement of the method as the pages describe it,
step by step, with numpy library primitives (matmul, exp, sort, cumsum) as
the only building blocks.  Source of the method (cited below as [GS]): the
gist.science summary page "Token Sparse Attention: Efficient Long-Context
Inference with Interleaved Token Selection" (arXiv 2602.03216), section
"2. Metodologia", sub-sections "Arquitectura Central" (compress, attend,
decompress per head) and "Cobertura Dinamica de Tokens" (proxy scoring,
budget, per-head selection).  The abstract pages with the same title
(chatpaper.ai, icml.cc poster 65647, fugumt.com) state the same
compress / attend / decompress scheme in summary form.

Readings taken where the page is silent (each is also pinned by a test):
  * "recent queries" = the last w query positions (all of them when the
    sequence is shorter than w); the proxy map is causal
    (window row at position i sees keys j <= i) and uses the attention's
    own scale 1/sqrt(d) (fp32 value, widened).
  * importance of key j = sum over the w window rows of the row-normalised
    proxy weights (the "vertical" sum); computed in fp64, rounded once to
    fp32 -- the fp32 score is the interface value both sides agree on.
  * coverage mass is measured exactly: q_j = ceil(score_j * 2^40) as int64,
    Q = sum q_j, threshold T = floor(tau * Q) in fp64 (tau is fp32).
    Tokens are taken in ascending q order; the pruned count p_h is the
    largest p whose first-p prefix sum stays <= T (the token that would
    push the pruned mass past tau is kept).  k_h = L - p_h.
  * the "global budget" is per sequence: k_b = max over heads of k_h
    (budget mode "max", the default).  Two variants the page leaves open:
    "mean" keeps k_b = ceil(mean over heads of k_h) in every head, and
    "per_head" keeps k_h in head h (no budget shared across heads).
  * optional forced keeps: with keep_recent = r, the last r tokens of the
    sequence are kept in every head; each k_h is raised to at least r, and
    the forced tokens rank above every score in the selection.
  * per-head top-k: the kept-count indices with the largest fp32 score,
    equal scores broken toward the smaller index, emitted in ascending order.
  * compressed causality: compressed row i attends compressed keys j <= i;
    since indices ascend, this is the original causal order.
  * GQA: selection per Q head h; K and V rows come from KV head h // G.
  * scatter: a zero L x d output per head; row S_h[i] receives row i of
    the compressed output; every other row is exactly zero.
  * block-sparse composition (optional): a block mask over 128-token blocks
    of compressed positions; compressed row i attends key j <= i only when
    j's block is i's own block or the mask allows the pair of blocks.

Every function here is pinned in ``tests/test_oracle_pins.py`` against brute
force, closed forms, hand-derived fixtures (``tests/golden``) and an
independent library routine (torch's fp64 scaled-dot-product attention).
"""
from __future__ import annotations

import numpy as np

from workloads import bf16_bits_to_f64

TWO_POW_40 = float(2 ** 40)


def default_scale(d: int) -> float:
    """Softmax scale: the fp32 value of 1/sqrt(d), widened to fp64."""
    return float(np.float32(1.0) / np.sqrt(np.float32(d)))


def _f64(x: np.ndarray) -> np.ndarray:
    if x.dtype == np.uint16:
        return bf16_bits_to_f64(x)
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Step 1: proxy attention map of the recent queries, summed per key column.
# [GS] "Cobertura Dinamica de Tokens", scoring bullet.
# ---------------------------------------------------------------------------
def proxy_scores_head(q_window: np.ndarray, k_head: np.ndarray, L: int, scale: float,
                      return_f64: bool = False):
    """Importance of every key of one head.

    q_window: [w, d] queries at positions L-w .. L-1; k_head: [L, d].
    Row r (position i = L-w+r) of the proxy map is the softmax over keys
    j <= i of scale * (q_i . k_j); the importance of key j is the sum of
    column j over the w rows.
    """
    qw = _f64(q_window)
    kh = _f64(k_head)
    w = qw.shape[0]
    x = (qw @ kh.T) * scale                                  # [w, L]
    pos = np.arange(L - w, L)[:, None]
    x = np.where(np.arange(L)[None, :] <= pos, x, -np.inf)   # causal proxy map
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    p = e / e.sum(axis=1, keepdims=True)                     # row softmax
    s64 = p.sum(axis=0)                                      # vertical sum
    s32 = s64.astype(np.float32)
    return (s32, s64) if return_f64 else s32


def proxy_scores(q, k, w: int, scale: float | None = None, return_f64: bool = False):
    """Scores [B, Hq, L] (fp32) for bf16 inputs q [B,Hq,L,d], k [B,Hkv,L,d]."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = default_scale(d)
    out = np.empty((B, Hq, L), dtype=np.float32)
    out64 = np.empty((B, Hq, L), dtype=np.float64) if return_f64 else None
    for b in range(B):
        for h in range(Hq):
            r = proxy_scores_head(q[b, h, max(L - w, 0):], k[b, h // G], L, scale, return_f64)
            if return_f64:
                out[b, h], out64[b, h] = r
            else:
                out[b, h] = r
    return (out, out64) if return_f64 else out


# ---------------------------------------------------------------------------
# Step 2: Dynamic Token Coverage budget.
# [GS] "Cobertura Dinamica de Tokens", budget bullet and per-head bullet.
# ---------------------------------------------------------------------------
def quantise_mass(scores: np.ndarray) -> np.ndarray:
    """Exact fixed-point mass: q = ceil(score * 2^40) as int64 (score >= 0)."""
    return np.ceil(np.asarray(scores, dtype=np.float32).astype(np.float64) * TWO_POW_40).astype(np.int64)


def coverage_threshold(qv: np.ndarray, tau: float) -> np.ndarray:
    """T = floor(tau * sum(q)) with tau as fp32 widened to fp64."""
    total = qv.sum(axis=-1)
    return np.floor(np.float64(np.float32(tau)) * total.astype(np.float64)).astype(np.int64)


def pruned_count_head(scores_head: np.ndarray, tau: float) -> int:
    """Largest p such that the p least important tokens carry mass <= T."""
    qv = quantise_mass(scores_head)
    T = int(coverage_threshold(qv, tau))
    cum = np.cumsum(np.sort(qv))            # ascending importance
    return int(np.count_nonzero(cum <= T))  # cum is non-decreasing


BUDGET_MODES = ("max", "mean", "per_head")


def coverage_budget(scores: np.ndarray, tau: float, mode: str = "max", keep_recent: int = 0):
    """Per-head keep counts k_h = max(L - p_h, r) [B,Hq] and the sequence
    budget k_b [B]: max over the heads ("max" and "per_head") or the ceiling
    of their mean ("mean").  r = keep_recent clipped to [0, L]."""
    if mode not in BUDGET_MODES:
        raise ValueError(mode)
    B, Hq, L = scores.shape
    r = min(max(int(keep_recent), 0), L)
    k_head = np.empty((B, Hq), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            k_head[b, h] = max(L - pruned_count_head(scores[b, h], tau), r)
    if mode == "mean":
        k_seq = -(-k_head.astype(np.int64).sum(axis=1) // Hq)   # ceiling of the mean
    else:
        k_seq = k_head.max(axis=1)                           # global budget of the sequence
    return k_head, k_seq.astype(np.int32)


def kept_counts(k_head: np.ndarray, k_seq: np.ndarray, mode: str = "max") -> np.ndarray:
    """Rows kept by every head [B,Hq]: its own k_h in "per_head" mode, else
    the sequence budget k_b."""
    if mode == "per_head":
        return np.asarray(k_head, dtype=np.int32).copy()
    return np.repeat(np.asarray(k_seq, dtype=np.int32)[:, None], k_head.shape[1], axis=1)


def _kept(kept: np.ndarray, b: int, h: int) -> int:
    """Kept rows of head (b, h) from per-sequence [B] or per-head [B,Hq] counts."""
    kept = np.asarray(kept)
    return int(kept[b] if kept.ndim == 1 else kept[b, h])


# ---------------------------------------------------------------------------
# Step 3: per-head top-k selection, ascending indices.
# [GS] "Cobertura Dinamica de Tokens", per-head selection bullet, and
# "Arquitectura Central", compression step.
# ---------------------------------------------------------------------------
def select_head(scores_head: np.ndarray, k: int, keep_recent: int = 0) -> np.ndarray:
    """The k best tokens, ascending: the last keep_recent tokens first, then
    score descending, then index ascending."""
    L = scores_head.shape[0]
    s = np.asarray(scores_head, dtype=np.float32).astype(np.float64)
    not_forced = np.arange(L) < L - min(max(int(keep_recent), 0), L)
    order = np.lexsort((np.arange(L), -s, not_forced))
    return np.sort(order[:k]).astype(np.int32)


def select_topk(scores: np.ndarray, kept: np.ndarray, keep_recent: int = 0) -> np.ndarray:
    """idx [B,Hq,L] int32: the first k entries of head (b, h) are S_h
    ascending, the rest -1; k comes from kept ([B] per sequence or [B,Hq]
    per head)."""
    B, Hq, L = scores.shape
    idx = np.full((B, Hq, L), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            kb = _kept(kept, b, h)
            idx[b, h, :kb] = select_head(scores[b, h], kb, keep_recent)
    return idx


# ---------------------------------------------------------------------------
# Step 4: gather into dense compressed tensors.  [GS] "Arquitectura Central".
# ---------------------------------------------------------------------------
def gather_qkv(q, k, v, idx, k_seq):
    """Compressed copies (same dtype as the inputs), rows >= k_b left zero.
    k_seq: kept rows per sequence [B] or per head [B,Hq]."""
    B, Hq, L, d = q.shape
    G = Hq // k.shape[1]
    qc = np.zeros_like(q)
    kc = np.zeros((B, Hq, L, d), dtype=k.dtype)
    vc = np.zeros((B, Hq, L, d), dtype=v.dtype)
    for b in range(B):
        for h in range(Hq):
            kb = _kept(k_seq, b, h)
            s = idx[b, h, :kb]
            qc[b, h, :kb] = q[b, h, s]
            kc[b, h, :kb] = k[b, h // G, s]
            vc[b, h, :kb] = v[b, h // G, s]
    return qc, kc, vc


# ---------------------------------------------------------------------------
# Step 5: causal attention over the compressed set.  [GS] "Arquitectura
# Central": the compressed tensors are attended by an ordinary dense kernel.
# ---------------------------------------------------------------------------
BLOCK = 128   # block edge of the block-sparse composition


def attention_rows(qc: np.ndarray, kc: np.ndarray, vc: np.ndarray, rows, scale: float,
                   chunk: int = 1024, block_mask: np.ndarray | None = None) -> np.ndarray:
    """Causal softmax attention for the listed rows of one head (fp64).

    Row i: o_i = sum_{j<=i, allowed} softmax_j(scale * q_i . k_j) v_j, where
    with a block mask [NB, NB] key j is allowed when j // 128 == i // 128 or
    block_mask[i // 128, j // 128] is nonzero (every key otherwise).
    Rows are evaluated independently; ``chunk`` only bounds memory.
    """
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.shape[0], vc.shape[-1]), dtype=np.float64)
    for c0 in range(0, rows.shape[0], chunk):
        r = rows[c0:c0 + chunk]
        n = int(r.max()) + 1
        qf = _f64(qc[r])
        kf = _f64(kc[:n])
        vf = _f64(vc[:n])
        x = (qf @ kf.T) * scale
        allow = np.arange(n)[None, :] <= r[:, None]
        if block_mask is not None:
            qb, kb = r[:, None] // BLOCK, np.arange(n)[None, :] // BLOCK
            allow &= (qb == kb) | (np.asarray(block_mask)[qb, kb] != 0)
        x = np.where(allow, x, -np.inf)
        m = x.max(axis=1, keepdims=True)
        e = np.exp(x - m)
        out[c0:c0 + chunk] = (e @ vf) / e.sum(axis=1, keepdims=True)
    return out


def compressed_attention(qc, kc, vc, k_seq, scale: float | None = None, block_mask=None) -> np.ndarray:
    """O_hat [B,Hq,L,d] fp64; rows >= k_b are zero.  block_mask: optional
    [B, Hq, NB, NB] over 128-token blocks of compressed positions."""
    B, Hq, L, d = qc.shape
    if scale is None:
        scale = default_scale(d)
    oc = np.zeros((B, Hq, L, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kb = _kept(k_seq, b, h)
            bm = None if block_mask is None else block_mask[b, h]
            oc[b, h, :kb] = attention_rows(qc[b, h, :kb], kc[b, h, :kb], vc[b, h, :kb],
                                           np.arange(kb), scale, block_mask=bm)
    return oc


def dense_causal_attention(q, k, v, scale: float | None = None) -> np.ndarray:
    """Dense causal GQA attention [B,Hq,L,d] fp64: the same row definition on
    the full sequence (the identity selection)."""
    B, Hq, L, d = q.shape
    G = Hq // k.shape[1]
    if scale is None:
        scale = default_scale(d)
    o = np.empty((B, Hq, L, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            o[b, h] = attention_rows(q[b, h], k[b, h // G], v[b, h // G], np.arange(L), scale)
    return o


# ---------------------------------------------------------------------------
# Step 6: scatter back into a zero-initialised full-length output.
# [GS] "Arquitectura Central", decompression step.
# ---------------------------------------------------------------------------
def scatter(oc: np.ndarray, idx: np.ndarray, k_seq: np.ndarray, L: int) -> np.ndarray:
    B, Hq, _, d = oc.shape
    o = np.zeros((B, Hq, L, d), dtype=oc.dtype)
    for b in range(B):
        for h in range(Hq):
            kb = _kept(k_seq, b, h)
            o[b, h, idx[b, h, :kb]] = oc[b, h, :kb]
    return o


# ---------------------------------------------------------------------------
# The whole path, step by step.
# ---------------------------------------------------------------------------
def forward(q, k, v, w: int, tau: float, scale: float | None = None, mode: str = "max",
            keep_recent: int = 0) -> dict:
    """Scores -> budget -> selection -> gather -> attention -> scatter."""
    B, Hq, L, d = q.shape
    if scale is None:
        scale = default_scale(d)
    scores = proxy_scores(q, k, w, scale)
    k_head, k_seq = coverage_budget(scores, tau, mode, keep_recent)
    kept = kept_counts(k_head, k_seq, mode)
    idx = select_topk(scores, kept, keep_recent)
    qc, kc, vc = gather_qkv(q, k, v, idx, kept)
    oc = compressed_attention(qc, kc, vc, kept, scale)
    o = scatter(oc, idx, kept, L)
    return dict(scores=scores, k_head=k_head, k_seq=k_seq, kept=kept, idx=idx, oc=oc, o=o)


def forward_varlen(q, k, v, cu_seqlens, w: int, tau: float, scale: float | None = None, mode: str = "max",
                   keep_recent: int = 0) -> list:
    """A batch of sequences of different lengths, packed token-major: q
    [T, Hq, d], k and v [T, Hkv, d], sequence b at tokens
    [cu_seqlens[b], cu_seqlens[b+1]).  Every sequence is independent, so each
    runs the whole path on its own; returns one ``forward`` result per
    sequence (arrays in the head-major layout of that sequence) and the
    packed output [T, Hq, d] under the key "o_packed" of the first."""
    cu = [int(c) for c in cu_seqlens]
    T, Hq, d = q.shape
    o_packed = np.zeros((T, Hq, d), dtype=np.float64)
    res = []
    for b in range(len(cu) - 1):
        t0, t1 = cu[b], cu[b + 1]
        hm = lambda x: np.ascontiguousarray(x[t0:t1].transpose(1, 0, 2))[None]   # [1, H, L_b, d]
        if t1 == t0:                              # an empty sequence keeps nothing
            z = np.zeros((1, Hq), dtype=np.int32)
            r = dict(scores=np.zeros((1, Hq, 0), np.float32), k_head=z, k_seq=np.zeros(1, np.int32), kept=z,
                     idx=np.zeros((1, Hq, 0), np.int32), oc=np.zeros((1, Hq, 0, d)), o=np.zeros((1, Hq, 0, d)))
            res.append(r)
            continue
        r = forward(hm(q), hm(k), hm(v), w, tau, scale, mode, min(keep_recent, t1 - t0))
        o_packed[t0:t1] = r["o"][0].transpose(1, 0, 2)
        res.append(r)
    if res:
        res[0]["o_packed"] = o_packed
    return res


def output_rows(q, k, v, idx, k_seq, b: int, h: int, orig_rows, scale: float | None = None):
    """Final output rows (original positions) of head (b, h), computed one by
    one from a given selection: zero if the position is not selected, else the
    compressed attention row.  Used to check large workloads by sampling."""
    B, Hq, L, d = q.shape
    G = Hq // k.shape[1]
    if scale is None:
        scale = default_scale(d)
    kb = _kept(k_seq, b, h)
    s = np.asarray(idx[b, h, :kb], dtype=np.int64)
    orig_rows = np.asarray(orig_rows, dtype=np.int64)
    pos = np.searchsorted(s, orig_rows)
    hit = (pos < kb) & (s[np.minimum(pos, kb - 1)] == orig_rows)
    out = np.zeros((orig_rows.shape[0], d), dtype=np.float64)
    if hit.any():
        cpos = pos[hit]
        n = int(cpos.max()) + 1
        sel = s[:n]
        out[hit] = attention_rows(q[b, h][sel], k[b, h // G][sel], v[b, h // G][sel], cpos, scale)
    return out
