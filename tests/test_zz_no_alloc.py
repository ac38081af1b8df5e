"""The allocation-free proxy-score entry point (tsa_score_noalloc).

It exists for callers that cannot call cudaMalloc (a plug-in whose framework
owns every device allocation, code under a hard memory budget, a C caller
without an allocator): it takes no workspace and keeps its scratch in a fixed
array inside the library.  It runs the same kernels as tsa_score on the same
inputs, so its output must equal tsa_score's bit for bit, and both must lie
within the score tolerance (1e-5 relative, element by element) of the fp64
oracle -- on two calls in a row with a different call in between (the array
keeps the previous call's contents, so this also checks that nothing stale is
read).  Its status word is read through tsa_score_noalloc_status, which needs
no workspace either.  This file is collected last so a failure here never
hides the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import token_sparse_attention_tsa_b200 as T
import workloads as W
from _gpu_util import scores_close

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).cuda()


def _case(wl):
    q, k, _ = W.generate(wl)
    return q, k, _dev(q), _dev(k), T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau)


def test_noalloc_scores_equal_workspace_scores_twice():
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(Hq=8, Hkv=2, L=3000, d=128, w=100, heavy_count=20, seed=21)
    wl2 = wl.with_(L=1500, w=64, seed=22)   # a different, smaller call in between
    outs = []
    for case in (wl, wl2, wl):
        q, k, dq, dk, p = _case(case)
        ws = T.new_workspace(p, full=False)
        ref = torch.empty((case.B, case.Hq, case.L), device="cuda")
        T.tsa_score(p, dq, dk, ref, ws)
        got = torch.full_like(ref, float("nan"))
        T.tsa_score_noalloc(p, dq, dk, got)
        assert T.score_noalloc_status() == (0, 0)
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32))       # same kernels: bit for bit
        _, s64 = O.proxy_scores(q, k, case.w, return_f64=True)
        assert scores_close(got.cpu().numpy(), s64) <= 1.0                     # 1e-5 relative
        outs.append(got.cpu().numpy())
    assert np.array_equal(outs[0].view(np.uint32), outs[2].view(np.uint32))   # same input, same output


def test_noalloc_reports_a_timeout_and_the_next_call_is_clean():
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(Hq=4, Hkv=2, L=2000, d=128, w=64, seed=23)
    q, k, dq, dk, p = _case(wl)
    stall = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, wl.tau, timeout_ms=50, flags=T.FLAG_TEST_STALL_SCORE)
    got = torch.full((wl.B, wl.Hq, wl.L), -3.0, device="cuda")
    T.tsa_score_noalloc(stall, dq, dk, got)
    st, flags = T.score_noalloc_status()
    assert st == TIMEOUT and flags & T.DEVFLAG_TIMEOUT
    assert (got == -3.0).all().item()          # the scores were not written
    # the next call clears the status word and is correct
    T.tsa_score_noalloc(p, dq, dk, got)
    assert T.score_noalloc_status() == (0, 0)
    _, s64 = O.proxy_scores(q, k, wl.w, return_f64=True)
    assert scores_close(got.cpu().numpy(), s64) <= 1.0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # scratch here: 8 x 64 heads x 4096 window rows x (12 bytes per key chunk + 8 bytes of row
    # statistics), over 40 MB, far beyond the 16 MiB array
    p = T.params(8, 64, 8, 1 << 21, 128, 4096, 0.05)
    assert T.stage_workspace_size(p) > T.NOALLOC_SCRATCH_BYTES
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")   # never touched: rejected on the host
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(T.TSAError) as e:
        T.tsa_score_noalloc(p, q, q, s)
    assert e.value.status == 3   # TSA_ERR_WORKSPACE
    rc = T.load().tsa_score_noalloc(ctypes.byref(p), None, None, None, None)
    assert rc == 1               # null pointers: TSA_ERR_INVALID_ARG
