"""Host-side tests of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before enqueuing any GPU work.

Every call here fails validation on the host, so none reaches a kernel; the
fake device addresses are never dereferenced.
"""
import ctypes
import os
import re

import pytest

import token_sparse_attention_tsa_b200 as T
from token_sparse_attention_tsa_b200 import build as tsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tsa.h")

FAKE = 0x7F0000000000   # 256-byte aligned, never dereferenced
INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    tsa_build.build()
    return T.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\*?\s+(tsa_[a-z_0-9]+)\(", text, re.M)))


def good(**kw):
    base = dict(B=1, Hq=8, Hkv=2, L=4096, d=128, w=64, tau=0.05)
    base.update(kw)
    return T.params(**base)


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) == len(T.EXPORTED) and set(names) == set(T.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.tsa_abi_version() == 3


def test_status_strings(lib):
    for code in range(8):
        assert lib.tsa_status_string(code)
    assert lib.tsa_status_string(99) == b"unknown status"


@pytest.mark.parametrize("kw,want", [
    (dict(), 0),
    (dict(B=0), INVALID), (dict(Hq=0), INVALID), (dict(L=0), INVALID), (dict(w=0), INVALID),
    (dict(Hq=6, Hkv=4), INVALID), (dict(w=5000, L=4096), INVALID), (dict(tau=1.0), INVALID),
    (dict(tau=-0.01), INVALID), (dict(tau=float("nan")), INVALID),
    (dict(softmax_scale=-1.0), INVALID), (dict(softmax_scale=float("inf")), INVALID),
    (dict(d=96), UNSUPPORTED), (dict(d=256), UNSUPPORTED), (dict(w=4097, L=8192), UNSUPPORTED),
    (dict(L=(1 << 22) + 1, w=1), UNSUPPORTED), (dict(B=64, Hq=64, Hkv=64, L=1 << 20), UNSUPPORTED),
    (dict(d=64), 0), (dict(w=1, L=1), 0), (dict(tau=0.0), 0),
    (dict(budget_mode=-1), INVALID), (dict(budget_mode=3), INVALID), (dict(budget_mode="mean"), 0),
    (dict(budget_mode="per_head"), 0), (dict(keep_recent=-1), INVALID), (dict(keep_recent=4097), INVALID),
    (dict(keep_recent=4096), 0), (dict(keep_recent=64, budget_mode="per_head"), 0),
    (dict(layout="blhd"), 0), (dict(layout=2), INVALID), (dict(layout=-1), INVALID),
    (dict(cu_seqlens=FAKE, total_tokens=9000), 0), (dict(cu_seqlens=FAKE, total_tokens=0), INVALID),
    (dict(cu_seqlens=FAKE + 2, total_tokens=10), INVALID), (dict(total_tokens=5), INVALID),
    (dict(cu_seqlens=FAKE, total_tokens=1 << 30), UNSUPPORTED),
])
def test_param_validation(lib, kw, want):
    p = good(**kw)
    assert T.check_params(p) == want


def test_flags_only_the_test_hook(lib):
    p = good()
    p.flags = 1
    assert T.check_params(p) == INVALID
    p.flags = T.FLAG_TEST_STALL
    assert T.check_params(p) == 0
    p.flags = T.FLAG_TEST_STALL_SCORE | T.FLAG_TEST_STALL
    assert T.check_params(p) == 0
    p.flags = T.FLAG_TEST_STALL_SCORE | 0x20000000
    assert T.check_params(p) == INVALID


def test_workspace_sizes(lib):
    p = good()
    full, stage = T.workspace_size(p), T.stage_workspace_size(p)
    assert stage < full
    # forward holds scores, indices and compressed Q, K and V (never a compressed output)
    assert p.B * p.Hq * p.L * (8 + 6 * p.d) <= full < p.B * p.Hq * p.L * (8 + 6 * p.d) + 2 * stage + 8192
    assert T.workspace_size(good(L=8192)) > full
    with pytest.raises(T.TSAError):
        T.workspace_size(good(d=96))


def _call(lib, name, *args):
    return getattr(lib, name)(*args)


def test_null_and_misaligned_pointers_rejected(lib):
    p = ctypes.byref(good())
    ws_n = T.stage_workspace_size(good())
    big = T.workspace_size(good())
    odd = FAKE + 8   # not 16-byte aligned
    # null tensor pointers
    assert _call(lib, "tsa_score", p, None, FAKE, FAKE, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_budget", p, FAKE, None, None, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_select", p, FAKE, FAKE, None, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_gather_qkv", p, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, None) == INVALID
    assert _call(lib, "tsa_attend", p, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_attend_dense", p, FAKE, FAKE, None, FAKE, None, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_scatter", p, FAKE, FAKE, FAKE, None, None, 0, None) == INVALID
    assert _call(lib, "tsa_attend_gathered", p, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_attend_gathered", p, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 64, None) == WORKSPACE
    assert _call(lib, "tsa_forward", p, FAKE, None, FAKE, FAKE, None, None, None, FAKE, big, None) == INVALID
    # misaligned tensors / workspace
    assert _call(lib, "tsa_score", p, odd, FAKE, FAKE, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_attend", p, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, FAKE, ws_n, None) == INVALID
    assert _call(lib, "tsa_forward", p, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE + 16, big, None) == INVALID
    assert _call(lib, "tsa_forward", p, FAKE, FAKE, FAKE, FAKE, odd, None, None, FAKE, big, None) == INVALID
    assert _call(lib, "tsa_reset_device_status", FAKE + 4, None) == INVALID
    assert _call(lib, "tsa_get_device_status", None, None, None) == INVALID


def test_layer_switch_arguments(lib):
    p = ctypes.byref(good())
    big = T.workspace_size(good())
    flags = (ctypes.c_uint8 * 4)(1, 0, 1, 0)
    fl = ctypes.cast(flags, ctypes.c_void_p)
    args = (FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, big, None)
    assert _call(lib, "tsa_layer_forward", p, 0, None, 4, *args) == INVALID      # no layer list
    assert _call(lib, "tsa_layer_forward", p, 4, fl, 4, *args) == INVALID        # layer out of range
    assert _call(lib, "tsa_layer_forward", p, -1, fl, 4, *args) == INVALID
    assert _call(lib, "tsa_layer_forward", p, 0, fl, 0, *args) == INVALID        # empty list
    # each branch reaches its own validation: sparse needs the full workspace,
    # dense only the stage workspace
    small = (FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, T.stage_workspace_size(good()), None)
    assert _call(lib, "tsa_layer_forward", p, 0, fl, 4, *small) == WORKSPACE
    assert _call(lib, "tsa_layer_forward", p, 1, fl, 4, FAKE, FAKE, None, FAKE, None, None, None, FAKE,
                 big, None) == INVALID                                          # dense branch: null v


def test_block_mask_call_arguments(lib):
    p = ctypes.byref(good())
    ws_n = T.stage_workspace_size(good())
    # qc, kc, vc, idx, k_seq, block_mask, o, lse, ws, ws_bytes, stream
    assert _call(lib, "tsa_attend_blocks", p, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, None, FAKE, ws_n,
                 None) == INVALID                                            # no mask
    assert _call(lib, "tsa_attend_blocks", p, FAKE, FAKE, FAKE, FAKE + 4, FAKE, FAKE, FAKE, None, FAKE, ws_n,
                 None) == INVALID                                            # misaligned idx
    assert _call(lib, "tsa_attend_blocks", p, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, FAKE, 8,
                 None) == WORKSPACE                                          # workspace too small
    assert _call(lib, "tsa_attend_blocks", None, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, FAKE, ws_n,
                 None) == INVALID                                            # no params


def test_per_head_budget_needs_head_counts(lib):
    p = ctypes.byref(good(budget_mode="per_head"))
    ws_n = T.stage_workspace_size(good(budget_mode="per_head"))
    assert _call(lib, "tsa_budget", p, FAKE, None, FAKE, FAKE, ws_n, None) == INVALID
    # the shared-budget modes accept a NULL k_head (scratch in the workspace)
    p_max = ctypes.byref(good())
    assert _call(lib, "tsa_budget", p_max, FAKE, None, FAKE, FAKE, 0, None) == WORKSPACE


def test_workspace_missing_or_small(lib):
    p = ctypes.byref(good())
    ws_n = T.stage_workspace_size(good())
    big = T.workspace_size(good())
    assert _call(lib, "tsa_score", p, FAKE, FAKE, FAKE, None, ws_n, None) == WORKSPACE
    assert _call(lib, "tsa_score", p, FAKE, FAKE, FAKE, FAKE, ws_n - 1, None) == WORKSPACE
    assert _call(lib, "tsa_budget", p, FAKE, FAKE, FAKE, FAKE, 0, None) == WORKSPACE
    assert _call(lib, "tsa_attend", p, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16, None) == WORKSPACE
    assert _call(lib, "tsa_forward", p, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, big - 256, None) == WORKSPACE
    # gather/scatter accept a NULL workspace but reject a too-small one
    assert _call(lib, "tsa_scatter", p, FAKE, FAKE, FAKE, FAKE, FAKE, 8, None) == WORKSPACE


def test_invalid_params_rejected_before_pointers(lib):
    p = ctypes.byref(good(d=96))
    assert _call(lib, "tsa_forward", p, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, 1 << 40, None) == UNSUPPORTED
    assert _call(lib, "tsa_score", None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == INVALID


def test_binding_refuses_cpu_tensors(lib):
    import torch
    p = good(L=256, w=8)
    q = torch.zeros((1, 8, 256, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        T.tsa_score(p, q, q, torch.zeros((1, 8, 256)), torch.zeros(16, dtype=torch.uint8))
