"""GPU check of the layer-level switch ([GS] section 2, "Seleccion de Capas
Dispersas"): a layer the caller marks sparse runs the token-sparse path, any
other layer dense causal attention.

Both kinds of layer are compared element by element with the CPU oracle:
  sparse  scores within 1e-5 relative of the fp64 oracle, budget and indices
          bit-exact from the GPU's scores, output within 2e-2 of
          oracle.scatter(oracle.compressed_attention(...)) on that selection
  dense   output within 2e-2 of oracle.dense_causal_attention
and a dense layer leaves the caller's intermediate buffers untouched."""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
from _gpu_util import bf16_to_f64, garbage_like, inputs, scores_close
from test_gpu_parity import ATOL_OUT, SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["gqa_d128_B2_L777_w130", "gqa_d64_L2500"])
def test_layer_switch_matches_the_oracle_per_layer(name):
    wl = SHAPES[name]
    (q, k, v), (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    ws = T.new_workspace(p, full=True)
    layers = [True, False, False, True]
    ref_dense = O.dense_causal_attention(q, k, v)
    _, s64 = O.proxy_scores(q, k, wl.w, return_f64=True)
    for layer, sparse in enumerate(layers):
        o = garbage_like(dq.shape)
        scores = torch.full((wl.B, wl.Hq, wl.L), -7.0, device="cuda")
        idx = torch.full((wl.B, wl.Hq, wl.L), -9, dtype=torch.int32, device="cuda")
        ks = torch.full((wl.B,), -5, dtype=torch.int32, device="cuda")
        T.tsa_layer_forward(p, layer, layers, dq, dk, dv, o, ws, scores_out=scores, idx_out=idx, k_seq_out=ks)
        got = bf16_to_f64(o)
        if not sparse:
            err = float(np.abs(got - ref_dense).max())
            assert err <= ATOL_OUT, (layer, err)
            # a dense layer leaves the intermediates alone
            assert (scores == -7.0).all().item() and (idx == -9).all().item() and (ks == -5).all().item()
            continue
        g_s, g_idx, g_ks = scores.cpu().numpy(), idx.cpu().numpy(), ks.cpu().numpy()
        assert scores_close(g_s, s64) <= 1.0, layer
        _, ref_ks = O.coverage_budget(g_s, wl.tau)
        assert np.array_equal(g_ks, ref_ks), layer
        assert np.array_equal(g_idx, O.select_topk(g_s, ref_ks)), layer
        qc, kc, vc = O.gather_qkv(q, k, v, g_idx, g_ks)
        ref = O.scatter(O.compressed_attention(qc, kc, vc, g_ks), g_idx, g_ks, wl.L)
        err = float(np.abs(got - ref).max())
        assert err <= ATOL_OUT, (layer, err)
        # unselected rows are exactly +0.0 (bit pattern 0)
        sel = np.zeros((wl.B, wl.Hq, wl.L), dtype=bool)
        for b in range(wl.B):
            for h in range(wl.Hq):
                sel[b, h, g_idx[b, h, :g_ks[b]]] = True
        bits = o.view(torch.int16).cpu().numpy()
        assert (bits[~sel] == 0).all(), layer
    assert_status_clean(ws)


def test_layer_switch_rejects_a_bad_layer_index():
    wl = SHAPES["mha_d128_L129"]
    _, (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    ws = T.new_workspace(p, full=True)
    o = garbage_like(dq.shape)
    for layer in (-1, 2):
        with pytest.raises(T.TSAError) as e:
            T.tsa_layer_forward(p, layer, [True, False], dq, dk, dv, o, ws)
        assert e.value.status == 1   # TSA_ERR_INVALID_ARG, nothing enqueued
    assert (o.view(torch.int16) == 0x7FC1).all().item()
