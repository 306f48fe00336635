"""Seeded synthetic inputs for the MXFP4 MoE layer.

This module only draws numbers: it holds none of the layer's arithmetic and
imports neither the oracle nor the CUDA library.  Both sides of every parity
check take their inputs from here.

Recipe (all draws from the counter-based generator in ``synth.cpp``):

====================  =======================  ======================================
tensor                distribution             substream (stream id, sub)
====================  =======================  ======================================
hidden x [T, d]       N(0, 1) -> bf16          (1, t | attempt << 32), one row each
RMSNorm weight [d]    N(1, 0.1) fp32           (2, 0)
router W [E, d]       N(0, 0.02) fp32          (3, 0)
router b [E]          N(0, 0.01) fp32          (4, 0)   (+ Zipf popularity term)
Zipf rank order       permutation of E         (5, 0)
W1 (gate_up) [2I, d]  N(0, 0.02) fp32 x w1_mul (6, e), one matrix per expert
W2 (down) [d, I]      N(0, 0.02) fp32          (7, e), one matrix per expert
====================  =======================  ======================================

The Zipf term (skewed-routing workload): expert e gets popularity rank
``rank_e = perm[e] + 1`` and its bias gains ``alpha * ln(rank_e^-s / H)`` with
``H = sum_r r^-s``, so the router prefers a few experts by a Zipf(s) law.

A hidden row can be redrawn (``attempt`` > 0) without touching any other value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.cpp")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None
_lock = threading.Lock()

STREAM_X, STREAM_GAMMA, STREAM_RW, STREAM_RB, STREAM_ZIPF, STREAM_W1, STREAM_W2 = 1, 2, 3, 4, 5, 6, 7


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (g++, C++17)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            u64, i64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
            L.synth_normal_f32.argtypes = [u64, u64, u64, u64, i64, dbl, dbl, vp, ctypes.c_int]
            L.synth_normal_bf16.argtypes = [u64, u64, u64, u64, i64, dbl, dbl, vp, ctypes.c_int]
            L.synth_uniform_f64.argtypes = [u64, u64, u64, u64, i64, vp]
            L.synth_permutation.argtypes = [u64, u64, u64, i32, vp]
            L.synth_u64.argtypes = [u64, u64, u64, u64, i64, vp]
            L.synth_splitmix64_sequence.argtypes = [u64, i64, vp]
            for f in (L.synth_normal_f32, L.synth_normal_bf16, L.synth_uniform_f64, L.synth_permutation,
                      L.synth_u64, L.synth_splitmix64_sequence):
                f.restype = None
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal_f32(seed, stream, sub, count, mean, std, offset=0, out=None, nthreads=0) -> np.ndarray:
    out = np.empty(count, np.float32) if out is None else out
    lib().synth_normal_f32(seed, stream, sub, offset, count, mean, std, _ptr(out), nthreads)
    return out


def normal_bf16(seed, stream, sub, count, mean, std, offset=0, out=None, nthreads=0) -> np.ndarray:
    out = np.empty(count, np.uint16) if out is None else out
    lib().synth_normal_bf16(seed, stream, sub, offset, count, mean, std, _ptr(out), nthreads)
    return out


def permutation(seed, stream, sub, n) -> np.ndarray:
    out = np.empty(n, np.int32)
    lib().synth_permutation(seed, stream, sub, n, _ptr(out))
    return out


def u64(seed, stream, sub, count, offset=0) -> np.ndarray:
    out = np.empty(count, np.uint64)
    lib().synth_u64(seed, stream, sub, offset, count, _ptr(out))
    return out


def splitmix64_sequence(seed, count) -> np.ndarray:
    out = np.empty(count, np.uint64)
    lib().synth_splitmix64_sequence(seed, count, _ptr(out))
    return out


@dataclass(frozen=True)
class MoEConfig:
    """One MoE-layer workload: shapes plus the input recipe's knobs."""
    name: str
    T: int
    d: int
    I: int
    E: int
    k: int
    zipf_s: float | None = None   # Zipf exponent of the router-bias popularity term
    zipf_alpha: float = 1.0       # multiplier of that term
    w1_mul: float = 1.0           # scales W1 (the clamp-stress case uses 8)
    seed: int = 0
    rms_eps: float = 1e-5
    swiglu_limit: float = 7.0

    @property
    def pairs(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


# The five workloads: a tiny layer, gpt-oss-20b at decode and prefill sizes,
# gpt-oss-120b, and a skewed-routing stress case at 120b width.
CONFIGS = {
    "tiny": MoEConfig("tiny", T=32, d=128, I=128, E=4, k=2),
    "decode_20b": MoEConfig("decode_20b", T=16, d=2880, I=2880, E=32, k=4),
    "prefill_20b": MoEConfig("prefill_20b", T=4096, d=2880, I=2880, E=32, k=4),
    "moe_120b": MoEConfig("moe_120b", T=8192, d=2880, I=2880, E=128, k=4),
    "skew_120b": MoEConfig("skew_120b", T=16384, d=2880, I=2880, E=128, k=4, zipf_s=1.2),
}


def hidden_rows(cfg: MoEConfig, rows, attempts=None) -> np.ndarray:
    """bf16 bit patterns [len(rows), d] of hidden rows ``rows`` at the given redraw attempts."""
    rows = np.asarray(rows, np.int64)
    attempts = np.zeros_like(rows) if attempts is None else np.asarray(attempts, np.int64)
    out = np.empty((len(rows), cfg.d), np.uint16)
    for i, (t, a) in enumerate(zip(rows.tolist(), attempts.tolist())):
        normal_bf16(cfg.seed, STREAM_X, (a << 32) | t, cfg.d, 0.0, 1.0, out=out[i], nthreads=1)
    return out


def hidden(cfg: MoEConfig, attempts=None) -> np.ndarray:
    """bf16 bit patterns [T, d]; ``attempts`` [T] selects each row's redraw (default 0)."""
    if attempts is None or not np.any(attempts):
        # Fast path: every row at attempt 0, generated row by row in parallel.
        out = np.empty((cfg.T, cfg.d), np.uint16)
        import concurrent.futures as cf
        def fill(lo, hi):
            for t in range(lo, hi):
                normal_bf16(cfg.seed, STREAM_X, t, cfg.d, 0.0, 1.0, out=out[t], nthreads=1)
        n = max(1, min(os.cpu_count() or 1, 16))
        step = (cfg.T + n - 1) // n
        with cf.ThreadPoolExecutor(n) as ex:
            list(ex.map(lambda i: fill(i * step, min(cfg.T, (i + 1) * step)), range(n)))
        return out
    return hidden_rows(cfg, np.arange(cfg.T), attempts)


def norm_weight(cfg: MoEConfig) -> np.ndarray:
    return normal_f32(cfg.seed, STREAM_GAMMA, 0, cfg.d, 1.0, 0.1)


def router_weight(cfg: MoEConfig) -> np.ndarray:
    return normal_f32(cfg.seed, STREAM_RW, 0, cfg.E * cfg.d, 0.0, 0.02).reshape(cfg.E, cfg.d)


def zipf_ranks(cfg: MoEConfig) -> np.ndarray:
    """Popularity rank (1 = most popular) of each expert."""
    return permutation(cfg.seed, STREAM_ZIPF, 0, cfg.E) + 1


def router_bias(cfg: MoEConfig) -> np.ndarray:
    b = normal_f32(cfg.seed, STREAM_RB, 0, cfg.E, 0.0, 0.01).astype(np.float64)
    if cfg.zipf_s is not None:
        r = zipf_ranks(cfg).astype(np.float64)
        H = np.sum(np.arange(1, cfg.E + 1, dtype=np.float64) ** -cfg.zipf_s)
        b = b + cfg.zipf_alpha * np.log(r ** -cfg.zipf_s / H)
    return b.astype(np.float32)


def w1_expert(cfg: MoEConfig, e: int, nthreads=0) -> np.ndarray:
    """fp32 [2I, d] gate_up weight of expert e: rows 0..I-1 gate, I..2I-1 up."""
    w = normal_f32(cfg.seed, STREAM_W1, e, 2 * cfg.I * cfg.d, 0.0, 0.02, nthreads=nthreads)
    if cfg.w1_mul != 1.0:
        w *= np.float32(cfg.w1_mul)
    return w.reshape(2 * cfg.I, cfg.d)


def w2_expert(cfg: MoEConfig, e: int, nthreads=0) -> np.ndarray:
    """fp32 [d, I] down weight of expert e."""
    return normal_f32(cfg.seed, STREAM_W2, e, cfg.d * cfg.I, 0.0, 0.02, nthreads=nthreads).reshape(cfg.d, cfg.I)


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)
