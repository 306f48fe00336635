"""Second, independent formulations used to pin the oracle (numpy, test-only).

The oracle runs experts sparsely (per expert, only its tokens, one dot product
at a time).  These formulations run *every* expert on *every* token as dense
matrix products and mask afterwards; MXFP4 is decoded from the bit fields of
the E2M1 format rather than from a table.
"""
from __future__ import annotations

import numpy as np


def e2m1_from_bits(code: int) -> float:
    """E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; exponent 0 is subnormal."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * m * 0.5
    return s * 2.0 ** (e - 1) * (1.0 + m / 2.0)


_E2M1 = np.array([e2m1_from_bits(c) for c in range(16)], np.float64)


def decode(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Oracle-layout MXFP4 [rows, K/2] + [rows, K/32] -> fp64 [rows, K] (vectorised)."""
    lo = codes & 0x0F
    hi = codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    vals = _E2M1[c]
    sc = np.exp2(scales.astype(np.float64) - 127.0)
    return vals * np.repeat(sc, 32, axis=1)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp64 to the nearest bfloat16 value, ties to even (vectorised, exact)."""
    v = np.asarray(v, np.float64)
    m, e = np.frexp(np.abs(v))
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    sub = np.abs(v) < 2.0 ** -126
    r = np.where(sub, np.rint(np.abs(v) * 2.0 ** 133) * 2.0 ** -133, r)
    return np.copysign(r, v)


def bf16_bits_to_f64(u16) -> np.ndarray:
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def silu(z):
    return z / (1.0 + np.exp(-z))


def dense_layer(x_bf16, gamma, rw, rb, w1_list, w2_list, k, eps=1e-5, limit=7.0, mode="topk"):
    """Every expert on every token; mix by top-k softmax (mode 'topk') or full softmax ('dense').

    w1_list[e]: fp64 [2I, d]; w2_list[e]: fp64 [d, I].  Returns (y fp64 before rounding, y rounded,
    logits, weights [T, E] with zeros off the selection).
    """
    x = bf16_bits_to_f64(x_bf16)
    T, d = x.shape
    E = len(w1_list)
    I = w1_list[0].shape[0] // 2
    ms = np.mean(x * x, axis=1, keepdims=True)
    xn = x / np.sqrt(ms + eps) * gamma.astype(np.float64)[None, :]
    logits = xn @ rw.astype(np.float64).T + (0.0 if rb is None else rb.astype(np.float64)[None, :])
    weights = np.zeros((T, E))
    if mode == "dense":
        z = np.exp(logits - logits.max(axis=1, keepdims=True))
        weights = z / z.sum(axis=1, keepdims=True)
        order = np.argsort(-logits, axis=1, kind="stable")
    else:
        order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
        sel = np.take_along_axis(logits, order, axis=1)
        z = np.exp(sel - sel[:, :1])
        np.put_along_axis(weights, order, z / z.sum(axis=1, keepdims=True), axis=1)
    xe = round_bf16(xn)
    outs = np.zeros((E, T, d))
    for e in range(E):
        gu = xe @ w1_list[e].T
        g, u = gu[:, :I], gu[:, I:]
        h = round_bf16(silu(np.minimum(g, limit)) * np.clip(u, -limit, limit))
        outs[e] = h @ w2_list[e].T
    # mix in the order of the selection (slot order), as the layer does
    y = x.copy()
    for j in range(order.shape[1]):
        e_j = order[:, j]
        y += weights[np.arange(T), e_j][:, None] * outs[e_j, np.arange(T)]
    return y, round_bf16(y), logits, weights
