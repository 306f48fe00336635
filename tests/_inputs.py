"""Test-side assembly of MoE-layer cases: synthetic inputs plus oracle-quantized weights.

Rejection of ambiguous routing: a token whose k-th and (k+1)-th router logits
(as the oracle computes them) differ by less than ``GAP_MIN`` has its hidden
row redrawn from the next generator attempt, until every token clears the gap.
Only the rows that need it change; everything else stays as generated.
"""
from __future__ import annotations

import functools

import numpy as np

import oracle
import synth

GAP_MIN = 1e-4
MAX_ATTEMPTS = 64


@functools.lru_cache(maxsize=4)
def routed_inputs(cfg: synth.MoEConfig, redraw: bool = True):
    """x (bf16 bits [T,d]), gamma, router W, router b, redraw attempts [T], oracle route of x."""
    x = synth.hidden(cfg)
    gamma = synth.norm_weight(cfg)
    rw = synth.router_weight(cfg)
    rb = synth.router_bias(cfg)
    attempts = np.zeros(cfg.T, np.int64)
    r = oracle.route(x, gamma, rw, rb, cfg.k, cfg.rms_eps)
    if redraw and cfg.k < cfg.E:
        for _ in range(MAX_ATTEMPTS):
            bad = np.nonzero(r["gap"] < GAP_MIN)[0]
            if len(bad) == 0:
                break
            attempts[bad] += 1
            x[bad] = synth.hidden_rows(cfg, bad, attempts[bad])
            rb_bad = oracle.route(x[bad], gamma, rw, rb, cfg.k, cfg.rms_eps)
            for key in ("idx", "w", "logits", "gap"):
                r[key][bad] = rb_bad[key]
        else:
            raise RuntimeError("gap redraw did not converge")
    return x, gamma, rw, rb, attempts, r


@functools.lru_cache(maxsize=2)
def oracle_weights(cfg: synth.MoEConfig, experts: tuple | None = None):
    """Oracle-layout MXFP4 weights of all experts (zeros for experts not in ``experts``).

    Returns (w1_codes [E,2I,d/2], w1_scales [E,2I,d/32], w2_codes [E,d,I/2], w2_scales [E,d,I/32]).
    """
    E, d, I = cfg.E, cfg.d, cfg.I
    w1c = np.zeros((E, 2 * I, d // 2), np.uint8)
    w1s = np.zeros((E, 2 * I, d // 32), np.uint8)
    w2c = np.zeros((E, d, I // 2), np.uint8)
    w2s = np.zeros((E, d, I // 32), np.uint8)
    for e in (range(E) if experts is None else experts):
        w1c[e], w1s[e] = oracle.quantize(synth.w1_expert(cfg, e))
        w2c[e], w2s[e] = oracle.quantize(synth.w2_expert(cfg, e))
    return w1c, w1s, w2c, w2s


def rel_frobenius(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_bits_to_f64(u16) -> np.ndarray:
    return synth.bf16_to_f32(u16).astype(np.float64)
