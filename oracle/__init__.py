"""CPU oracle of the MXFP4 MoE layer (ctypes front end of ``moe_oracle.cpp``).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``mxfp4_expert_gemm_b200``) never imports it.

Every function here is argument marshalling; the arithmetic lives in the C++
file, which cites the passages it follows.  The oracle's weight layout is its
own: codes [rows][K/2] (low nibble = even k), scale bytes [rows][K/32].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O2, strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC", "-pthread",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            i32, i64, dbl, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            L.oracle_mxfp4_code_bytes.argtypes = [i64, i32]
            L.oracle_mxfp4_code_bytes.restype = i64
            L.oracle_mxfp4_scale_bytes.argtypes = [i64, i32]
            L.oracle_mxfp4_scale_bytes.restype = i64
            L.oracle_e2m1_value.argtypes = [i32]
            L.oracle_e2m1_value.restype = dbl
            L.oracle_quantize.argtypes = [vp, i64, i32, vp, vp]
            L.oracle_quantize.restype = i32
            L.oracle_dequantize.argtypes = [vp, vp, i64, i32, vp]
            L.oracle_dequantize.restype = i32
            L.oracle_round_bf16.argtypes = [dbl]
            L.oracle_round_bf16.restype = dbl
            L.oracle_to_bf16.argtypes = [vp, i64, vp]
            L.oracle_to_bf16.restype = None
            L.oracle_rmsnorm.argtypes = [i32, i32, vp, vp, dbl, vp]
            L.oracle_rmsnorm.restype = None
            L.oracle_route.argtypes = [i32, i32, i32, i32, vp, vp, dbl, vp, vp, vp, vp, vp, vp, i32]
            L.oracle_route.restype = None
            L.oracle_group.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
            L.oracle_group.restype = i32
            L.oracle_moe_forward.argtypes = [i32, i32, i32, i32, i32, dbl, dbl, vp, vp, vp, vp, vp, vp, vp, vp,
                                             vp, i32, vp, vp, vp, vp, vp, i32, i32]
            L.oracle_moe_forward.restype = i32
            L.oracle_e4m3_nearest_code.argtypes = [dbl]
            L.oracle_e4m3_nearest_code.restype = i32
            L.oracle_e4m3_value.argtypes = [i32]
            L.oracle_e4m3_value.restype = dbl
            L.oracle_mxfp4_quantize_values.argtypes = [vp, i64, vp]
            L.oracle_mxfp4_quantize_values.restype = i32
            L.oracle_mxfp8_quantize.argtypes = [vp, i64, vp, vp]
            L.oracle_mxfp8_quantize.restype = i32
            _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "contiguous numpy array expected"
    return a.ctypes.data


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(code)


def round_bf16(v: float) -> float:
    return lib().oracle_round_bf16(float(v))


# Activation formats of the expert GEMMs: bf16 (exact), MXFP8 (E4M3 in 32-blocks) or MXFP4
# (E2M1 in 32-blocks, the weights' own format).
ACT_FORMATS = {"bf16": 0, "mxfp8": 1, "mxfp4": 2}


def e4m3_nearest_code(a: float) -> int:
    """E4M3 code (0..0x7E) of the value nearest to |a|; ties to the even code; saturating."""
    return lib().oracle_e4m3_nearest_code(float(a))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def mxfp8_quantize(v: np.ndarray):
    """float64 [..., n] (n a multiple of 32) -> (quantized values, block exponents [..., n/32])."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty_like(v)
    exps = np.empty(v.shape[:-1] + (v.shape[-1] // 32,), np.int32)
    if lib().oracle_mxfp8_quantize(_p(v), v.size, _p(out), _p(exps)):
        raise ValueError("length is not a multiple of 32")
    return out, exps


def mxfp4_quantize_values(v: np.ndarray) -> np.ndarray:
    """float64 [..., n] (n a multiple of 32) -> the values after MXFP4 quantization in
    32-value blocks, by the rule the expert weights are quantized with."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty_like(v)
    if lib().oracle_mxfp4_quantize_values(_p(v), v.size, _p(out)):
        raise ValueError("length is not a multiple of 32")
    return out


def storage_bytes(rows: int, K: int) -> tuple[int, int]:
    """(code bytes, scale bytes) of an MXFP4 matrix [rows][K]."""
    return lib().oracle_mxfp4_code_bytes(rows, K), lib().oracle_mxfp4_scale_bytes(rows, K)


def quantize(w: np.ndarray):
    """fp32 [rows, K] -> (codes [rows, K/2] u8, scale bytes [rows, K/32] u8)."""
    w = np.ascontiguousarray(w, np.float32)
    rows, K = w.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    st = lib().oracle_quantize(_p(w), rows, K, _p(codes), _p(scales))
    if st:
        raise ValueError(f"oracle_quantize status {st} (non-finite input)")
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), np.float64)
    st = lib().oracle_dequantize(_p(codes), _p(scales), rows, K, _p(out))
    if st:
        raise ValueError("NaN scale byte")
    return out


def rmsnorm(x_bf16: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    gamma = np.ascontiguousarray(gamma, np.float32)
    T, d = x_bf16.shape
    out = np.empty((T, d), np.float64)
    lib().oracle_rmsnorm(T, d, _p(x_bf16), _p(gamma), eps, _p(out))
    return out


def to_bf16(v: np.ndarray) -> np.ndarray:
    """float64 array -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_to_bf16(_p(v), v.size, _p(out))
    return out


def next_block_norm(y_bf16: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """The next block's first RMSNorm of a block's bf16 output, rounded to bf16 (every block
    holds two RMSNorms; ewbang.com GPT-OSS article, section Transformer 块)."""
    return to_bf16(rmsnorm(y_bf16, gamma, eps))


def route(x_bf16, gamma, router_w, router_b, k, eps, nthreads=0):
    """-> dict(idx [T,k] i32, w [T,k] f64, logits [T,E] f64, gap [T] f64)."""
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    gamma = np.ascontiguousarray(gamma, np.float32)
    router_w = np.ascontiguousarray(router_w, np.float32)
    rb = None if router_b is None else np.ascontiguousarray(router_b, np.float32)
    T, d = x_bf16.shape
    E = router_w.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    logits = np.empty((T, E), np.float64)
    gap = np.empty(T, np.float64)
    lib().oracle_route(T, d, E, k, _p(x_bf16), _p(gamma), eps, _p(router_w), _p(rb), _p(idx), _p(w), _p(logits),
                       _p(gap), nthreads)
    return dict(idx=idx, w=w, logits=logits, gap=gap)


def group(idx: np.ndarray, E: int):
    """-> dict(counts [E], offsets [E+1], perm [P], inv [P]) (all int32)."""
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    st = lib().oracle_group(T, k, E, _p(idx), _p(counts), _p(offsets), _p(perm), _p(inv))
    if st:
        raise ValueError("invalid expert indices")
    return dict(counts=counts, offsets=offsets, perm=perm, inv=inv)


def moe_forward(x_bf16, gamma, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, *, I, k,
                eps=1e-5, limit=7.0, tokens=None, want_h=False, nthreads=0, act="bf16"):
    """The whole layer for ``tokens`` (default: all rows of x).

    Weights in the oracle layout with a leading expert axis:
    w1_codes [E, 2I, d/2], w1_scales [E, 2I, d/32], w2_codes [E, d, I/2], w2_scales [E, d, I/32].
    act: "bf16" (exact bf16 activations), "mxfp8" or "mxfp4" (the expert inputs and the SwiGLU
    outputs quantized to E4M3 / E2M1 in 32-value blocks before each projection; h is then
    returned quantized).
    Returns dict(y bf16 bits [n,d], y_f64 [n,d], idx [n,k], w [n,k], h [n,k,I] bf16 bits or None).
    """
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    T, d = x_bf16.shape
    E = router_w.shape[0]
    toks = None if tokens is None else np.ascontiguousarray(tokens, np.int32)
    n = T if toks is None else len(toks)
    y = np.empty((n, d), np.uint16)
    y64 = np.empty((n, d), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    h = np.empty((n, k, I), np.uint16) if want_h else None
    args = [np.ascontiguousarray(a) for a in (gamma, router_w)]
    rb = None if router_b is None else np.ascontiguousarray(router_b, np.float32)
    st = lib().oracle_moe_forward(
        T, d, I, E, k, eps, limit, _p(x_bf16), _p(np.ascontiguousarray(gamma, np.float32)),
        _p(np.ascontiguousarray(router_w, np.float32)), _p(rb),
        _p(np.ascontiguousarray(w1_codes, np.uint8)), _p(np.ascontiguousarray(w1_scales, np.uint8)),
        _p(np.ascontiguousarray(w2_codes, np.uint8)), _p(np.ascontiguousarray(w2_scales, np.uint8)),
        _p(toks), n, _p(y), _p(y64), _p(idx), _p(w), _p(h), nthreads, ACT_FORMATS[act])
    del args
    if st:
        raise ValueError(f"oracle_moe_forward status {st}")
    return dict(y=y, y_f64=y64, idx=idx, w=w, h=h)
