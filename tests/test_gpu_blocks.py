"""GPU parity of attention with a block-sparse mask over the compressed
sequence (tsa_attend_blocks) against the oracle.

An all-ones mask must reproduce the unmasked kernel bit for bit; random,
block-local and "sink + local band" masks are compared with the oracle's
masked compressed attention on every row; a mask whose two query tiles of a
CTA pair attend different key tiles exercises the all-zero P path.
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, from_dev_bf16, garbage_like, inputs
from test_gpu_parity import ATOL_OUT, SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu


def compressed_setup(name, mode="max"):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, budget_mode=mode)
    ws = T.new_workspace(p, full=True)
    o = garbage_like(dq.shape)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    kept = torch.empty((wl.B, wl.Hq) if mode == "per_head" else (wl.B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, kept)
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    qc, kc, vc = (garbage_like(shape) for _ in range(3))
    T.tsa_gather_qkv(p, dq, dk, dv, idx, kept, qc, kc, vc, ws)
    return wl, p, ws, (q, k, v), (qc, kc, vc), o, idx, kept


def masks(wl, seed):
    nb = (wl.L + 127) // 128
    rng = np.random.default_rng(seed)
    shape = (wl.B, wl.Hq, nb, nb)
    ii, jj = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    band = ((ii - jj) <= 2) | (jj == 0)                 # sink block + a local band
    alternating = np.broadcast_to((ii % 2 == 0) & (jj == 0), (nb, nb))   # pair tiles disagree on block 0
    return {
        "random_half": (rng.random(shape) < 0.5).astype(np.uint8),
        "random_sparse": (rng.random(shape) < 0.15).astype(np.uint8),
        "block_local": np.zeros(shape, np.uint8),
        "sink_band": np.broadcast_to(band, shape).astype(np.uint8).copy(),
        "pair_disagree": np.broadcast_to(alternating, shape).astype(np.uint8).copy(),
    }


@pytest.mark.parametrize("name,mode", [("gqa_d128_B2_L777_w130", "max"), ("gqa_d64_L2500", "per_head"),
                                       ("mha_d128_L129", "max")])
def test_all_ones_mask_equals_unmasked(name, mode):
    wl, p, ws, _, (qc, kc, vc), o, idx, kept = compressed_setup(name, mode)
    nb = (wl.L + 127) // 128
    ones = torch.ones((wl.B, wl.Hq, nb, nb), dtype=torch.uint8, device="cuda")
    oc_ref, oc = garbage_like(qc.shape), garbage_like(qc.shape)
    T.tsa_attend(p, qc, kc, vc, kept, oc_ref, None, ws)
    T.tsa_attend_blocks(p, qc, kc, vc, None, kept, ones, oc, None, ws)
    kn = kept.cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.Hq):
            n = int(kn[b, h] if kn.ndim == 2 else kn[b])
            assert torch.equal(oc[b, h, :n].view(torch.int16), oc_ref[b, h, :n].view(torch.int16))
    o2 = garbage_like(o.shape)
    T.tsa_attend_blocks(p, qc, kc, vc, idx, kept, ones, o2, None, ws)
    assert torch.equal(o2.view(torch.int16), o.view(torch.int16))
    assert_status_clean(ws)


@pytest.mark.parametrize("mask_name", ["random_half", "random_sparse", "block_local", "sink_band", "pair_disagree"])
@pytest.mark.parametrize("name,mode", [("gqa_d128_B2_L777_w130", "per_head"), ("gqa_d64_L2500", "max")])
def test_masked_attention_matches_oracle(name, mode, mask_name):
    wl, p, ws, (q, k, v), (qc, kc, vc), _, idx, kept = compressed_setup(name, mode)
    bm = masks(wl, seed=len(mask_name))[mask_name]
    dbm = torch.from_numpy(bm).cuda()
    g_idx, kn = idx.cpu().numpy(), kept.cpu().numpy()
    kr = kn if kn.ndim == 2 else np.repeat(kn[:, None], wl.Hq, axis=1)
    qn, kcn, vcn = O.gather_qkv(q, k, v, g_idx, kr)
    ref = O.compressed_attention(qn, kcn, vcn, kr, block_mask=bm)
    # compressed output
    oc = garbage_like(qc.shape)
    T.tsa_attend_blocks(p, qc, kc, vc, None, kept, dbm, oc, None, ws)
    got = bf16_to_f64(oc)
    for b in range(wl.B):
        for h in range(wl.Hq):
            n = int(kr[b, h])
            assert np.abs(got[b, h, :n] - ref[b, h, :n]).max() <= ATOL_OUT, (b, h)
    # scattered output, unselected rows exactly zero
    o = garbage_like((wl.B, wl.Hq, wl.L, wl.d))
    T.tsa_attend_blocks(p, qc, kc, vc, idx, kept, dbm, o, None, ws)
    full = O.scatter(ref, g_idx, kr, wl.L)
    assert np.abs(bf16_to_f64(o) - full).max() <= ATOL_OUT
    o16 = from_dev_bf16(o)
    for b in range(wl.B):
        for h in range(wl.Hq):
            unsel = np.setdiff1d(np.arange(wl.L), g_idx[b, h, :kr[b, h]])
            assert (o16[b, h, unsel] == 0).all()
    assert_status_clean(ws)


def test_sink_band_mask_32k_sampled():
    """The 32K workload with a sink + local band mask: sampled rows against
    the oracle's masked attention evaluated row by row."""
    wl = W.WORKLOADS["c3_L32K_gqa_band"]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(dq)
    scores = torch.empty((wl.B, wl.Hq, wl.L), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device="cuda")
    ks = torch.empty((wl.B,), dtype=torch.int32, device="cuda")
    T.tsa_forward(p, dq, dk, dv, o, ws, scores, idx, ks)
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    qc, kc, vc = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    T.tsa_gather_qkv(p, dq, dk, dv, idx, ks, qc, kc, vc, ws)
    nb = (wl.L + 127) // 128
    ii, jj = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    band = (((ii - jj) <= 8) | (jj == 0)).astype(np.uint8)
    bm = np.broadcast_to(band, (wl.B, wl.Hq, nb, nb)).copy()
    ob = torch.empty_like(dq)
    T.tsa_attend_blocks(p, qc, kc, vc, idx, ks, torch.from_numpy(bm).cuda(), ob, None, ws)
    assert T.get_device_status(ws)[0] == 0
    g_idx, kb = idx.cpu().numpy(), int(ks.cpu()[0])
    rng = np.random.default_rng(4)
    scale = O.default_scale(wl.d)
    for h in (0, 31):
        S = g_idx[0, h, :kb].astype(np.int64)
        crow = np.unique(np.concatenate([[0, 127, 128, 1151, 1152, kb - 1], rng.integers(0, kb, 6)]))
        qs, kss, vs = q[0, h][S], k[0, h // wl.G][S], v[0, h // wl.G][S]
        ref = O.attention_rows(qs, kss, vs, crow, scale, block_mask=band)
        got = bf16_to_f64(ob[0, h, torch.from_numpy(S[crow]).cuda()])
        assert np.abs(got - ref).max() <= ATOL_OUT, h
