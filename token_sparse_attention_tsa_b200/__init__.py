"""Token Sparse Attention prefill path on NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/tsa.h`` (``libtsa.so`` beside
this file).  The functions here only marshal torch tensors into pointers and
the current CUDA stream; every step of the path runs in the library's CUDA
kernels.  There is no CPU fallback: if the library is missing or the tensors
are not on a CUDA device, the calls raise.

Names follow the C ABI: ``tsa_score``, ``tsa_budget``, ``tsa_select``,
``tsa_gather_qkv``, ``tsa_attend``, ``tsa_attend_dense``, ``tsa_scatter``,
``tsa_forward``, plus workspace and status helpers.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtsa.so")

TSA_OK = 0
STATUS_NAMES = {0: "TSA_OK", 1: "TSA_ERR_INVALID_ARG", 2: "TSA_ERR_UNSUPPORTED", 3: "TSA_ERR_WORKSPACE",
                4: "TSA_ERR_CUDA", 5: "TSA_ERR_NONFINITE", 6: "TSA_ERR_TIMEOUT", 7: "TSA_ERR_BAD_INDEX"}
DEVFLAG_NONFINITE, DEVFLAG_TIMEOUT, DEVFLAG_BAD_INDEX = 0x1, 0x2, 0x4
FLAG_TEST_STALL = 0x80000000
FLAG_TEST_STALL_SCORE = 0x40000000
BUDGET_MAX, BUDGET_MEAN, BUDGET_PER_HEAD = 0, 1, 2
BUDGET_MODES = {"max": BUDGET_MAX, "mean": BUDGET_MEAN, "per_head": BUDGET_PER_HEAD}
LAYOUT_BHLD, LAYOUT_BLHD = 0, 1
LAYOUTS = {"bhld": LAYOUT_BHLD, "blhd": LAYOUT_BLHD}

# Every symbol the header declares (checked by the tests).
EXPORTED = ("tsa_abi_version", "tsa_status_string", "tsa_check_params", "tsa_workspace_size",
            "tsa_stage_workspace_size", "tsa_reset_device_status", "tsa_get_device_status",
            "tsa_score", "tsa_budget", "tsa_select", "tsa_gather_qkv", "tsa_attend",
            "tsa_attend_dense", "tsa_attend_scatter", "tsa_attend_gathered", "tsa_attend_blocks", "tsa_scatter",
            "tsa_forward", "tsa_forward_begin", "tsa_forward_end", "tsa_layer_forward", "tsa_score_noalloc",
            "tsa_score_noalloc_status")


class TSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_string(status)})")


class tsa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("L", ctypes.c_int32), ("d", ctypes.c_int32), ("w", ctypes.c_int32),
                ("tau", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("flags", ctypes.c_uint32), ("timeout_ms", ctypes.c_uint32),
                ("budget_mode", ctypes.c_int32), ("keep_recent", ctypes.c_int32), ("layout", ctypes.c_int32),
                ("total_tokens", ctypes.c_int32), ("cu_seqlens", ctypes.c_void_p)]


def params(B, Hq, Hkv, L, d, w, tau, softmax_scale=0.0, timeout_ms=0, flags=0, budget_mode=BUDGET_MAX,
           keep_recent=0, layout=LAYOUT_BHLD, cu_seqlens=None, total_tokens=0) -> tsa_params:
    """budget_mode: BUDGET_MAX / BUDGET_MEAN / BUDGET_PER_HEAD or "max" / "mean" / "per_head".
    layout: LAYOUT_BHLD / LAYOUT_BLHD or "bhld" / "blhd" (memory order of q, k, v, o).
    cu_seqlens: for a packed varlen batch, a CUDA int32 tensor [B+1] (kept
    alive by the caller while the params are used), with total_tokens = T
    and L = the longest sequence; the layout is then token-major."""
    if isinstance(budget_mode, str):
        budget_mode = BUDGET_MODES[budget_mode]
    if isinstance(layout, str):
        layout = LAYOUTS[layout]
    cu = None
    if cu_seqlens is not None:
        cu = cu_seqlens if isinstance(cu_seqlens, int) else _ptr(cu_seqlens, "cu_seqlens", _torch().int32)
        layout = LAYOUT_BLHD
    return tsa_params(B, Hq, Hkv, L, d, w, tau, softmax_scale, flags, timeout_ms, budget_mode, keep_recent, layout,
                      total_tokens, cu)


def _torch():
    import torch
    return torch


_lock = threading.Lock()
_lib = None

_P = ctypes.POINTER(tsa_params)
_v = ctypes.c_void_p
_sz = ctypes.c_size_t


def load(path: str | None = None):
    """Load ``libtsa.so`` (raises if it is absent: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise FileNotFoundError(f"{p} is missing; build it with token_sparse_attention_tsa_b200/build.py")
        lib = ctypes.CDLL(p)
        sig = {
            "tsa_abi_version": ([], ctypes.c_int32),
            "tsa_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "tsa_check_params": ([_P], ctypes.c_int),
            "tsa_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
            "tsa_stage_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
            "tsa_reset_device_status": ([_v, _v], ctypes.c_int),
            "tsa_get_device_status": ([_v, _v, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
            "tsa_score": ([_P, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_budget": ([_P, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_select": ([_P, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_gather_qkv": ([_P, _v, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_attend": ([_P, _v, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_attend_dense": ([_P, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_attend_gathered": ([_P, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_attend_scatter": ([_P, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_attend_blocks": ([_P, _v, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_scatter": ([_P, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_forward": ([_P, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_forward_begin": ([_P, _v, _v, _v, _v, _v, _v, _sz, _v], ctypes.c_int),
            "tsa_forward_end": ([_P, ctypes.c_int32, _v, _v, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v],
                                ctypes.c_int),
            "tsa_layer_forward": ([_P, ctypes.c_int32, _v, ctypes.c_int32, _v, _v, _v, _v, _v, _v, _v, _v, _sz, _v],
                                  ctypes.c_int),
            "tsa_score_noalloc": ([_P, _v, _v, _v, _v], ctypes.c_int),
            "tsa_score_noalloc_status": ([_v, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def _string(status: int) -> str:
    try:
        return load().tsa_status_string(status).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(status: int, where: str):
    if status != TSA_OK:
        raise TSAError(status, where)


def _ptr(t, name: str, dtype=None):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


# ---------------------------------------------------------------- sizing
def workspace_size(p: tsa_params) -> int:
    n = _sz()
    _check(load().tsa_workspace_size(ctypes.byref(p), ctypes.byref(n)), "tsa_workspace_size")
    return n.value


def stage_workspace_size(p: tsa_params) -> int:
    n = _sz()
    _check(load().tsa_stage_workspace_size(ctypes.byref(p), ctypes.byref(n)), "tsa_stage_workspace_size")
    return n.value


def check_params(p: tsa_params) -> int:
    """Status code of the host-side validation (no exception)."""
    return load().tsa_check_params(ctypes.byref(p))


def new_workspace(p: tsa_params, full: bool = True, device=None):
    """A uint8 CUDA tensor sized for tsa_forward (full) or the stage calls,
    with its status word cleared."""
    import torch
    n = workspace_size(p) if full else stage_workspace_size(p)
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    reset_device_status(ws)
    return ws


def reset_device_status(ws, stream=None):
    _check(load().tsa_reset_device_status(_ptr(ws, "ws"), _stream(stream)), "tsa_reset_device_status")


def get_device_status(ws, stream=None) -> tuple[int, int]:
    """(status code, raw flag bits) of the device status word; synchronises."""
    flags = ctypes.c_uint32()
    st = load().tsa_get_device_status(_ptr(ws, "ws"), _stream(stream), ctypes.byref(flags))
    return st, flags.value


# ---------------------------------------------------------------- stages
def tsa_score(p, q, k, scores, ws, stream=None):
    import torch
    _check(load().tsa_score(ctypes.byref(p), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                            _ptr(scores, "scores", torch.float32), _ptr(ws, "ws"), _nbytes(ws),
                            _stream(stream)), "tsa_score")


NOALLOC_SCRATCH_BYTES = 16 << 20   # TSA_NOALLOC_SCRATCH_BYTES of the header


def tsa_score_noalloc(p, q, k, scores, stream=None):
    """tsa_score for callers that cannot allocate device memory: no workspace;
    the library's fixed 16 MiB device scratch is used instead (one call at a
    time per device; the first call on a device must precede stream capture)."""
    import torch
    _check(load().tsa_score_noalloc(ctypes.byref(p), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                    _ptr(scores, "scores", torch.float32), _stream(stream)), "tsa_score_noalloc")


def score_noalloc_status(stream=None) -> tuple[int, int]:
    """(status code, raw flag bits) of the most recent tsa_score_noalloc call
    on the current device; synchronises."""
    flags = ctypes.c_uint32()
    st = load().tsa_score_noalloc_status(_stream(stream), ctypes.byref(flags))
    return st, flags.value


def tsa_budget(p, scores, k_head, k_seq, ws, stream=None):
    import torch
    _check(load().tsa_budget(ctypes.byref(p), _ptr(scores, "scores", torch.float32),
                             _ptr(k_head, "k_head", torch.int32), _ptr(k_seq, "k_seq", torch.int32),
                             _ptr(ws, "ws"), _nbytes(ws), _stream(stream)), "tsa_budget")


def tsa_select(p, scores, k_seq, idx, ws, stream=None):
    import torch
    _check(load().tsa_select(ctypes.byref(p), _ptr(scores, "scores", torch.float32),
                             _ptr(k_seq, "k_seq", torch.int32), _ptr(idx, "idx", torch.int32),
                             _ptr(ws, "ws"), _nbytes(ws), _stream(stream)), "tsa_select")


def tsa_gather_qkv(p, q, k, v, idx, k_seq, qc, kc, vc, ws=None, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_gather_qkv(ctypes.byref(p), _ptr(q, "q", bf), _ptr(k, "k", bf), _ptr(v, "v", bf),
                                 _ptr(idx, "idx", torch.int32), _ptr(k_seq, "k_seq", torch.int32),
                                 _ptr(qc, "qc", bf), _ptr(kc, "kc", bf), _ptr(vc, "vc", bf),  # qc may be None
                                 _ptr(ws, "ws"), _nbytes(ws) if ws is not None else 0, _stream(stream)),
           "tsa_gather_qkv")


def tsa_attend(p, qc, kc, vc, k_seq, oc, lse, ws, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_attend(ctypes.byref(p), _ptr(qc, "qc", bf), _ptr(kc, "kc", bf), _ptr(vc, "vc", bf),
                             _ptr(k_seq, "k_seq", torch.int32), _ptr(oc, "oc", bf),
                             _ptr(lse, "lse", torch.float32), _ptr(ws, "ws"), _nbytes(ws), _stream(stream)),
           "tsa_attend")


def tsa_attend_dense(p, q, k, v, o, lse, ws, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_attend_dense(ctypes.byref(p), _ptr(q, "q", bf), _ptr(k, "k", bf), _ptr(v, "v", bf),
                                   _ptr(o, "o", bf), _ptr(lse, "lse", torch.float32), _ptr(ws, "ws"),
                                   _nbytes(ws), _stream(stream)), "tsa_attend_dense")


def tsa_attend_scatter(p, qc, kc, vc, idx, k_seq, o, lse, ws, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_attend_scatter(ctypes.byref(p), _ptr(qc, "qc", bf), _ptr(kc, "kc", bf), _ptr(vc, "vc", bf),
                                     _ptr(idx, "idx", torch.int32), _ptr(k_seq, "k_seq", torch.int32),
                                     _ptr(o, "o", bf), _ptr(lse, "lse", torch.float32), _ptr(ws, "ws"),
                                     _nbytes(ws), _stream(stream)), "tsa_attend_scatter")


def tsa_attend_blocks(p, qc, kc, vc, idx, k_seq, block_mask, o, lse, ws, stream=None):
    """idx None: compressed output in o; else o in the caller's layout."""
    import torch
    bf = torch.bfloat16
    _check(load().tsa_attend_blocks(ctypes.byref(p), _ptr(qc, "qc", bf), _ptr(kc, "kc", bf), _ptr(vc, "vc", bf),
                                    _ptr(idx, "idx", torch.int32), _ptr(k_seq, "k_seq", torch.int32),
                                    _ptr(block_mask, "block_mask", torch.uint8), _ptr(o, "o", bf),
                                    _ptr(lse, "lse", torch.float32), _ptr(ws, "ws"), _nbytes(ws),
                                    _stream(stream)), "tsa_attend_blocks")


def tsa_attend_gathered(p, q, k, v, idx, k_seq, o, lse, ws, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_attend_gathered(ctypes.byref(p), _ptr(q, "q", bf), _ptr(k, "k", bf), _ptr(v, "v", bf),
                                      _ptr(idx, "idx", torch.int32), _ptr(k_seq, "k_seq", torch.int32),
                                      _ptr(o, "o", bf), _ptr(lse, "lse", torch.float32), _ptr(ws, "ws"),
                                      _nbytes(ws), _stream(stream)), "tsa_attend_gathered")


def tsa_scatter(p, oc, idx, k_seq, o, ws=None, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_scatter(ctypes.byref(p), _ptr(oc, "oc", bf), _ptr(idx, "idx", torch.int32),
                              _ptr(k_seq, "k_seq", torch.int32), _ptr(o, "o", bf), _ptr(ws, "ws"),
                              _nbytes(ws) if ws is not None else 0, _stream(stream)), "tsa_scatter")


def tsa_forward(p, q, k, v, o, ws, scores_out=None, idx_out=None, k_seq_out=None, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_forward(ctypes.byref(p), _ptr(q, "q", bf), _ptr(k, "k", bf), _ptr(v, "v", bf),
                              _ptr(o, "o", bf), _ptr(scores_out, "scores_out", torch.float32),
                              _ptr(idx_out, "idx_out", torch.int32), _ptr(k_seq_out, "k_seq_out", torch.int32),
                              _ptr(ws, "ws"), _nbytes(ws), _stream(stream)), "tsa_forward")


def tsa_forward_begin(p, q, k, k_part, ws, scores_out=None, k_head_out=None, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_forward_begin(ctypes.byref(p), _ptr(q, "q", bf), _ptr(k, "k", bf),
                                    _ptr(scores_out, "scores_out", torch.float32),
                                    _ptr(k_head_out, "k_head_out", torch.int32), _ptr(k_part, "k_part", torch.int32),
                                    _ptr(ws, "ws"), _nbytes(ws), _stream(stream)), "tsa_forward_begin")


def tsa_forward_end(p, Hq_total: int, q, k, v, o, k_reduced, ws, scores=None, k_head=None, idx_out=None,
                    k_seq_out=None, stream=None):
    import torch
    bf = torch.bfloat16
    _check(load().tsa_forward_end(ctypes.byref(p), int(Hq_total), _ptr(q, "q", bf), _ptr(k, "k", bf),
                                  _ptr(v, "v", bf), _ptr(o, "o", bf), _ptr(scores, "scores", torch.float32),
                                  _ptr(k_head, "k_head", torch.int32), _ptr(k_reduced, "k_reduced", torch.int32),
                                  _ptr(idx_out, "idx_out", torch.int32), _ptr(k_seq_out, "k_seq_out", torch.int32),
                                  _ptr(ws, "ws"), _nbytes(ws), _stream(stream)), "tsa_forward_end")


# ---------------------------------------------------------------- head sharding
def budget_reduce_op(budget_mode) -> str | None:
    """How the budget partials of tsa_forward_begin combine over the devices
    that share a sequence's heads: "max" (MAX mode), "sum" (MEAN mode: the
    partials are count sums) or None (PER_HEAD mode: nothing is shared)."""
    if isinstance(budget_mode, str):
        budget_mode = BUDGET_MODES[budget_mode]
    return {BUDGET_MAX: "max", BUDGET_MEAN: "sum", BUDGET_PER_HEAD: None}[budget_mode]


def shard_heads(Hq: int, Hkv: int, world: int, rank: int) -> tuple[int, int, int, int]:
    """Heads of `rank` when a sequence's Hq query heads are split evenly over
    `world` devices: query heads [h0, h1) and the key/value heads [kv0, kv1)
    they read (query head h reads KV head h // (Hq // Hkv)).  Each device
    holds whole GQA groups, or a whole divisor of one group (its KV head is
    then also held by the other devices of that group)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if Hq % Hkv or Hq % world:
        raise ValueError(f"Hq={Hq} must be divisible by Hkv={Hkv} and by world={world}")
    G = Hq // Hkv
    n = Hq // world
    if n % G and G % n:
        raise ValueError(f"{n} query heads per device split a group of {G} unevenly")
    h0, h1 = rank * n, (rank + 1) * n
    return h0, h1, h0 // G, (h1 - 1) // G + 1


def forward_sharded(p, Hq_total: int, q, k, v, o, ws, group=None, scores_out=None, idx_out=None, k_seq_out=None,
                    k_part=None):
    """The forward of this device's heads of a head-sharded batch (p, q, k, v,
    o describe the local heads; Hq_total counts a sequence's query heads over
    all devices): tsa_forward_begin, one all-reduce of the B budget partials
    over `group` (torch.distributed, e.g. NCCL; skipped when nothing is
    shared or the group has one member), tsa_forward_end.  Runs on the
    current CUDA stream.  k_part: optional int32 [B] buffer for the partials
    (allocated when None); returned after the exchange."""
    import torch
    import torch.distributed as dist
    if k_part is None:
        k_part = torch.empty((p.B,), dtype=torch.int32, device=q.device)
    tsa_forward_begin(p, q, k, k_part, ws, scores_out=scores_out)
    op = budget_reduce_op(p.budget_mode)
    if op is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(k_part, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM, group=group)
    tsa_forward_end(p, Hq_total, q, k, v, o, k_part, ws, scores=scores_out, idx_out=idx_out, k_seq_out=k_seq_out)
    return k_part


def tsa_layer_forward(p, layer: int, sparse_layers, q, k, v, o, ws, scores_out=None, idx_out=None, k_seq_out=None,
                      stream=None):
    """sparse_layers: a sequence of per-layer flags (host side), e.g. a list
    of bools; layer selects this call's entry."""
    import torch
    bf = torch.bfloat16
    flags = (ctypes.c_uint8 * len(sparse_layers))(*[1 if x else 0 for x in sparse_layers])
    _check(load().tsa_layer_forward(ctypes.byref(p), int(layer), ctypes.cast(flags, ctypes.c_void_p),
                                    len(sparse_layers), _ptr(q, "q", bf), _ptr(k, "k", bf), _ptr(v, "v", bf),
                                    _ptr(o, "o", bf), _ptr(scores_out, "scores_out", torch.float32),
                                    _ptr(idx_out, "idx_out", torch.int32),
                                    _ptr(k_seq_out, "k_seq_out", torch.int32), _ptr(ws, "ws"), _nbytes(ws),
                                    _stream(stream)), "tsa_layer_forward")


def forward(q, k, v, w: int, tau: float, softmax_scale: float = 0.0, ws=None, return_intermediates=False,
            budget_mode=BUDGET_MAX, keep_recent: int = 0, layout="bhld"):
    """Convenience wrapper: allocate the output (and workspace if not given)
    and run ``tsa_forward`` on the current stream.  q, k, v are [B, H, L, d]
    (layout "bhld") or [B, L, H, d] ("blhd"); o comes back in the same
    layout.  With intermediates, the kept counts come back as [B], or
    [B, Hq] in the per-head budget mode."""
    import torch
    if isinstance(layout, str):
        layout = LAYOUTS[layout]
    if layout == LAYOUT_BLHD:
        B, L, Hq, d = q.shape
        Hkv = k.shape[2]
    else:
        B, Hq, L, d = q.shape
        Hkv = k.shape[1]
    p = params(B, Hq, Hkv, L, d, w, tau, softmax_scale, budget_mode=budget_mode, keep_recent=keep_recent,
               layout=layout)
    if ws is None:
        ws = new_workspace(p, full=True, device=q.device)
    o = torch.empty_like(q)
    if not return_intermediates:
        tsa_forward(p, q, k, v, o, ws)
        return o
    scores = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    idx = torch.empty((B, Hq, L), dtype=torch.int32, device=q.device)
    kshape = (B, Hq) if p.budget_mode == BUDGET_PER_HEAD else (B,)
    k_seq = torch.empty(kshape, dtype=torch.int32, device=q.device)
    tsa_forward(p, q, k, v, o, ws, scores, idx, k_seq)
    return o, scores, idx, k_seq


def forward_varlen(q, k, v, cu_seqlens, max_seqlen: int, w: int, tau: float, softmax_scale: float = 0.0,
                   ws=None, return_intermediates=False, budget_mode=BUDGET_MAX, keep_recent: int = 0):
    """Convenience wrapper for a packed varlen batch: q [T, Hq, d], k and v
    [T, Hkv, d], cu_seqlens a CUDA int32 tensor [B+1] of token offsets and
    max_seqlen the longest sequence.  Returns o [T, Hq, d] (and, with
    intermediates, scores, idx, kept as in ``forward`` with capacity
    max_seqlen)."""
    import torch
    T_tok, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    p = params(B, Hq, Hkv, max_seqlen, d, w, tau, softmax_scale, budget_mode=budget_mode,
               keep_recent=keep_recent, cu_seqlens=cu_seqlens, total_tokens=T_tok)
    if ws is None:
        ws = new_workspace(p, full=True, device=q.device)
    o = torch.empty_like(q)
    if not return_intermediates:
        tsa_forward(p, q, k, v, o, ws)
        return o
    scores = torch.empty((B, Hq, max_seqlen), dtype=torch.float32, device=q.device)
    idx = torch.empty((B, Hq, max_seqlen), dtype=torch.int32, device=q.device)
    kshape = (B, Hq) if p.budget_mode == BUDGET_PER_HEAD else (B,)
    kept = torch.empty(kshape, dtype=torch.int32, device=q.device)
    tsa_forward(p, q, k, v, o, ws, scores, idx, kept)
    return o, scores, idx, kept
