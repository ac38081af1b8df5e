"""GPU check of the layer-level switch: a layer the caller marks sparse runs
the token-sparse path, any other layer dense causal attention, bit for bit
the same as calling those paths directly."""
import pytest
import torch

import token_sparse_attention_tsa_b200 as T
from _gpu_util import garbage_like, inputs
from test_gpu_parity import SHAPES, assert_status_clean

pytestmark = pytest.mark.gpu


def test_layer_switch_dispatches_per_layer():
    wl = SHAPES["gqa_d128_B2_L777_w130"]
    _, (dq, dk, dv) = inputs(wl)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)
    ws = T.new_workspace(p, full=True)
    layers = [True, False, False, True]
    o_sparse, o_dense = garbage_like(dq.shape), garbage_like(dq.shape)
    T.tsa_forward(p, dq, dk, dv, o_sparse, ws)
    T.tsa_attend_dense(p, dq, dk, dv, o_dense, None, ws)
    for layer, sparse in enumerate(layers):
        o = garbage_like(dq.shape)
        idx = torch.full((wl.B, wl.Hq, wl.L), -9, dtype=torch.int32, device="cuda")
        T.tsa_layer_forward(p, layer, layers, dq, dk, dv, o, ws, idx_out=idx)
        ref = o_sparse if sparse else o_dense
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), layer
        if not sparse:
            assert (idx == -9).all().item()            # dense layers leave the intermediates alone
        else:
            assert (idx[:, :, 0] >= -1).all().item()
    assert_status_clean(ws)
