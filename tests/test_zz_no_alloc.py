"""The allocation-free proxy-score entry point (tsa_score_noalloc).

It exists for callers that cannot call cudaMalloc (a plug-in whose framework
owns every device allocation, code under a hard memory budget, a C caller
without an allocator): it takes no workspace and keeps its scratch in a fixed
array inside the library.  Its output must match tsa_score, which takes the
same scratch from a caller workspace, on two calls in a row (the array keeps
the previous call's contents, so the second call checks that nothing stale is
read).  This file is collected last so a failure here never hides the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import token_sparse_attention_tsa_b200 as T
import workloads as W

pytestmark = pytest.mark.gpu

SCORE_RTOL = 1e-5   # the score tolerance used by the parity tests


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).cuda()


def test_noalloc_scores_match_workspace_scores_twice():
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(Hq=8, Hkv=2, L=3000, d=128, w=100, heavy_count=20, seed=21)
    wl2 = wl.with_(L=1500, w=64, seed=22)   # a different, smaller call in between
    outs = []
    for case in (wl, wl2, wl):
        q, k, _ = (_dev(x) for x in W.generate(case))
        p = T.params(case.B, case.Hq, case.Hkv, case.L, case.d, case.w, case.tau)
        ws = T.new_workspace(p, full=False)
        ref = torch.empty((case.B, case.Hq, case.L), device="cuda")
        T.tsa_score(p, q, k, ref, ws)
        got = torch.full_like(ref, float("nan"))
        T.tsa_score_noalloc(p, q, k, got)
        torch.cuda.synchronize()
        r, g = ref.cpu().numpy().astype(np.float64), got.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - r) <= SCORE_RTOL * np.abs(r) + 1e-30)
        outs.append(g)
    assert np.array_equal(outs[0], outs[2])   # same input, same output after another call


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # scratch here: 64 heads x 4096 window rows x 4096 key chunks x 12 bytes, far over 16 MiB
    p = T.params(1, 64, 8, 1 << 22, 128, 4096, 0.05)
    assert T.stage_workspace_size(p) > T.NOALLOC_SCRATCH_BYTES
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")   # never touched: rejected on the host
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(T.TSAError) as e:
        T.tsa_score_noalloc(p, q, q, s)
    assert e.value.status == 3   # TSA_ERR_WORKSPACE
    rc = T.load().tsa_score_noalloc(ctypes.byref(p), None, None, None, None)
    assert rc == 1               # null pointers: TSA_ERR_INVALID_ARG
