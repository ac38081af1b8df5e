"""Seeded synthetic workloads for the Token Sparse Attention prefill path.

This module only draws inputs; it holds none of the method's arithmetic.
The generator itself is C (``gen.c``, compiled to ``libtsagen.so`` beside
this file) so that the 128K-token workloads are produced in seconds; both the
CPU oracle and the CUDA path read the same bf16 bytes from it.

The workload shapes follow the long-context prefill evaluation of the Token
Sparse Attention pages (LLaMA-3.1-8B / Mistral-Nemo style heads, 8K to 128K
tokens).  The benchmark suites those pages use (RULER, InfiniteBench,
Needle-in-a-Haystack) are not available here; these synthetic tensors stand
in for them: N(0,1) bf16 values with planted heavy keys, an optional sink at
position 0 and an optional local band correlation between Q and K.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libtsagen.so")
_lock = threading.Lock()
_lib = None


class _Spec(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("L", ctypes.c_int32), ("d", ctypes.c_int32),
        ("seed", ctypes.c_uint64),
        ("heavy_count", ctypes.c_int32),
        ("heavy_frac_lo", ctypes.c_double), ("heavy_frac_hi", ctypes.c_double),
        ("heavy_scale", ctypes.c_float),
        ("sink", ctypes.c_int32), ("sink_scale", ctypes.c_float),
        ("band_half", ctypes.c_int32), ("band_a", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile ``gen.c`` into ``libtsagen.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.tsagen_generate.argtypes = [ctypes.POINTER(_Spec), ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p]
            lib.tsagen_generate.restype = ctypes.c_int
            lib.tsagen_heavy_rows.argtypes = [ctypes.POINTER(_Spec), ctypes.c_int32,
                                              ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32]
            lib.tsagen_heavy_rows.restype = ctypes.c_int32
            lib.tsagen_mix64.argtypes = [ctypes.c_uint64]
            lib.tsagen_mix64.restype = ctypes.c_uint64
            lib.tsagen_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
            lib.tsagen_draw.restype = ctypes.c_uint64
            lib.tsagen_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
            lib.tsagen_normal.restype = ctypes.c_double
            lib.tsagen_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.tsagen_f32_to_bf16.restype = ctypes.c_uint16
            _lib = lib
    return _lib


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, method parameters and input recipe of one prefill workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    w: int
    tau: float
    seed: int
    heavy_count: int = 0
    heavy_frac_lo: float = 0.0
    heavy_frac_hi: float = 0.0
    heavy_scale: float = 1.0
    sink: bool = False
    sink_scale: float = 1.0
    band_half: int = 0
    band_a: float = 0.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def spec(self) -> _Spec:
        return _Spec(self.B, self.Hq, self.Hkv, self.L, self.d, self.seed,
                     self.heavy_count, self.heavy_frac_lo, self.heavy_frac_hi,
                     self.heavy_scale, int(self.sink), self.sink_scale,
                     self.band_half, self.band_a)

    def describe(self) -> dict:
        return dataclasses.asdict(self)


# The five workloads the method is measured on.  Heavy keys are planted per
# (sequence, KV head): K is shared inside a GQA group, so "per head" is read
# as per KV head; the Q heads of a group still differ through their own Q.
WORKLOADS = {
    # MHA, 1K tokens, d=64: key 0 and 16 random keys x4.
    "c1_L1K_mha_d64": Workload("c1_L1K_mha_d64", B=1, Hq=4, Hkv=4, L=1024, d=64, w=32,
                               tau=0.05, seed=1, heavy_count=16, heavy_scale=4.0,
                               sink=True, sink_scale=4.0),
    # MHA 32 heads, 8K tokens: 1% heavy keys x3.
    "c2_L8K_mha": Workload("c2_L8K_mha", B=1, Hq=32, Hkv=32, L=8192, d=128, w=64, tau=0.05,
                           seed=2, heavy_frac_lo=0.01, heavy_frac_hi=0.01, heavy_scale=3.0),
    # GQA 32/8, 32K tokens: 0.5% heavy keys x3 plus a +-128 local band (a=0.5).
    "c3_L32K_gqa_band": Workload("c3_L32K_gqa_band", B=1, Hq=32, Hkv=8, L=32768, d=128, w=64,
                                 tau=0.1, seed=3, heavy_frac_lo=0.005, heavy_frac_hi=0.005,
                                 heavy_scale=3.0, band_half=128, band_a=0.5),
    # GQA 32/8, 128K tokens: 0.25% heavy keys x3 and a x4 sink at position 0.
    "c4_L128K_gqa": Workload("c4_L128K_gqa", B=1, Hq=32, Hkv=8, L=131072, d=128, w=128,
                             tau=0.05, seed=4, heavy_frac_lo=0.0025, heavy_frac_hi=0.0025,
                             heavy_scale=3.0, sink=True, sink_scale=4.0),
    # 4 sequences of 64K, GQA 28/4: heavy fraction U[0.1%, 2%] per KV head.
    "c5_B4_L64K_gqa": Workload("c5_B4_L64K_gqa", B=4, Hq=28, Hkv=4, L=65536, d=128, w=128,
                               tau=0.05, seed=5, heavy_frac_lo=0.001, heavy_frac_hi=0.02,
                               heavy_scale=3.0),
}

C4_TAU_SWEEP = (0.01, 0.05, 0.1)


def generate(wl: Workload):
    """Return (q, k, v) as uint16 numpy arrays holding bf16 bit patterns.

    q is [B, Hq, L, d]; k and v are [B, Hkv, L, d]; all C-contiguous.
    """
    lib = _load()
    q = np.empty((wl.B, wl.Hq, wl.L, wl.d), dtype=np.uint16)
    k = np.empty((wl.B, wl.Hkv, wl.L, wl.d), dtype=np.uint16)
    v = np.empty((wl.B, wl.Hkv, wl.L, wl.d), dtype=np.uint16)
    spec = wl.spec()
    rc = lib.tsagen_generate(ctypes.byref(spec), q.ctypes.data, k.ctypes.data, v.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"tsagen_generate failed ({rc}) for {wl.name}")
    return q, k, v


def heavy_rows(wl: Workload, b: int, g: int) -> np.ndarray:
    """The heavy K rows planted in (sequence b, KV head g)."""
    lib = _load()
    spec = wl.spec()
    cap = wl.L
    out = np.empty(cap, dtype=np.int32)
    m = lib.tsagen_heavy_rows(ctypes.byref(spec), b, g, out.ctypes.data, cap)
    if m < 0:
        raise RuntimeError("tsagen_heavy_rows failed")
    return out[:m].copy()


def bf16_bits_to_f64(x: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    return (x.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (vectorised)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def raw():
    """The loaded C library (for tests that pin the generator)."""
    return _load()
