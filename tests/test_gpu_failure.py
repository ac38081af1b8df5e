"""Failure detection on the GPU without a fault: a pipeline wait that runs out.

With TSA_FLAG_TEST_STALL the attention kernel's MMA issuer first waits on a
barrier that nothing completes.  Its bounded wait expires after timeout_ms;
the kernel records TSA_DEVFLAG_TIMEOUT in the workspace status word, lets
its in-flight copies land, frees its tensor memory and returns.  The host
reads the status, and the same context then runs normal calls correctly.
"""
import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import bf16_to_f64, garbage_like, inputs

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS["c1_L1K_mha_d64"].with_(Hq=4, Hkv=2, L=1500, d=128, w=40, seed=31)
TIMEOUT = 6


def _params(**kw):
    return T.params(WL.B, WL.Hq, WL.Hkv, WL.L, WL.d, WL.w, WL.tau, **kw)


def test_attention_wait_runs_out_and_context_survives():
    (q, k, v), (dq, dk, dv) = inputs(WL)
    stall = _params(timeout_ms=50, flags=T.FLAG_TEST_STALL)
    ws = T.new_workspace(stall, full=False)
    o = garbage_like(dq.shape)
    T.tsa_attend_dense(stall, dq, dk, dv, o, None, ws)
    st, flags = T.get_device_status(ws)
    assert st == TIMEOUT and flags & T.DEVFLAG_TIMEOUT
    # nothing was written: the output still holds its fill pattern
    assert (o.view(torch.int16) == 0x7FC1).all().item()
    # the context is intact: a normal call on the same stream is correct
    T.reset_device_status(ws)
    T.tsa_attend_dense(_params(), dq, dk, dv, o, None, ws)
    assert T.get_device_status(ws) == (0, 0)
    rows = np.array([0, 1, 700, WL.L - 1])
    for h in (0, WL.Hq - 1):
        ref = O.attention_rows(q[0, h], k[0, h // WL.G], v[0, h // WL.G], rows, O.default_scale(WL.d))
        got = bf16_to_f64(o[0, h, torch.from_numpy(rows).cuda()])
        assert np.abs(got - ref).max() <= 2e-2


def test_forward_reports_timeout_then_recovers():
    (q, k, v), (dq, dk, dv) = inputs(WL)
    stall = _params(timeout_ms=50, flags=T.FLAG_TEST_STALL)
    ws = T.new_workspace(stall, full=True)
    o = torch.empty_like(dq)
    T.tsa_forward(stall, dq, dk, dv, o, ws)
    st, flags = T.get_device_status(ws)
    assert st == TIMEOUT and flags & T.DEVFLAG_TIMEOUT
    T.reset_device_status(ws)
    out, scores, idx, k_seq = T.forward(dq, dk, dv, WL.w, WL.tau, ws=ws, return_intermediates=True)
    assert T.get_device_status(ws) == (0, 0)
    g_idx, g_ks = idx.cpu().numpy(), k_seq.cpu().numpy()
    qc, kc, vc = O.gather_qkv(q, k, v, g_idx, g_ks)
    ref = O.scatter(O.compressed_attention(qc, kc, vc, g_ks), g_idx, g_ks, WL.L)
    assert np.abs(bf16_to_f64(out) - ref).max() <= 2e-2


def test_score_wait_runs_out_and_context_survives():
    """TSA_FLAG_TEST_STALL_SCORE: the proxy-score kernel's bounded wait runs
    out; the stage call and the forward report TIMEOUT (whatever else the
    later steps flag on the unwritten scores), and normal calls that follow
    on the same context are correct."""
    (q, k, v), (dq, dk, dv) = inputs(WL)
    stall = _params(timeout_ms=50, flags=T.FLAG_TEST_STALL_SCORE)
    ws = T.new_workspace(stall, full=True)
    scores = torch.full((WL.B, WL.Hq, WL.L), -3.0, device="cuda")
    T.tsa_score(stall, dq, dk, scores, ws)
    st, flags = T.get_device_status(ws)
    assert st == TIMEOUT and flags & T.DEVFLAG_TIMEOUT
    assert (scores == -3.0).all().item()          # not written
    T.reset_device_status(ws)
    o = torch.empty_like(dq)
    T.tsa_forward(stall, dq, dk, dv, o, ws)
    st, flags = T.get_device_status(ws)
    assert st == TIMEOUT and flags & T.DEVFLAG_TIMEOUT
    T.reset_device_status(ws)
    T.tsa_score(_params(), dq, dk, scores, ws)
    assert T.get_device_status(ws) == (0, 0)
    _, s64 = O.proxy_scores(q, k, WL.w, return_f64=True)
    err = np.abs(scores.cpu().numpy().astype(np.float64) - s64)
    assert (err <= 1e-5 * np.abs(s64) + 1e-30).all()
