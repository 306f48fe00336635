"""GPU-side assembly of parity cases (test infrastructure).

Inputs come from ``synth``; the library quantizes the fp32 weights on the GPU and
the oracle quantizes the same fp32 weights on the CPU, expert by expert, so the
two sides share nothing but the generator.  The GPU's codes and scales are
compared with the oracle's bit for bit as they are produced.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import mxfp4_expert_gemm_b200 as moe
import oracle
import synth
from _inputs import routed_inputs


# Token tile of each path (moe_mxfp4.h: "8-token tiles", "96-token tiles"; twice that with
# MXFP8 activations, one MMA column per token).
TILE_TOKENS = {"gemv": 8, "gemm": 96}


def tile_tokens(path: str, act: str = "bf16") -> int:
    return TILE_TOKENS[path] * (1 if act == "bf16" else 2)


_E2M1_LUT = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])


def decode_e2m1_packed(b: np.ndarray) -> np.ndarray:
    """Packed E2M1 bytes -> float64 values, two per byte (element 2i in the low nibble)."""
    b = b.astype(np.int64)
    return np.stack([_E2M1_LUT[b & 15], _E2M1_LUT[b >> 4]], axis=-1).reshape(*b.shape[:-1], -1)


def decode_e4m3(b: np.ndarray) -> np.ndarray:
    """E4M3 bytes -> float64 from the format's fields: sign bit 7, exponent bits 6..3
    (bias 7), mantissa bits 2..0; exponent 0 is subnormal (m/8 * 2^-6); 0x7F / 0xFF NaN."""
    b = b.astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 15
    m = (b & 7).astype(np.float64)
    v = np.where(e == 0, m / 8 * 2.0 ** -6, (1 + m / 8) * np.exp2(e.astype(np.float64) - 7))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return sign * v


def stored_row_of(N: int, role: str) -> np.ndarray:
    """Stored row of each logical row n: gate_up tensors pair 64 gate rows with the 64
    matching up rows in every 128-row tile; other tensors keep their order."""
    n = np.arange(N)
    if role != "gate_up":
        return n
    I = N // 2
    part = (n >= I).astype(np.int64)
    f = n - part * I
    return (f // 64) * 128 + part * 64 + f % 64


def stored_to_rowmajor(codes: np.ndarray, scales: np.ndarray, N: int, K: int, role: str):
    """Library MXFP4 storage -> the oracle's row-major layout.

    codes [E, NT, KC, 128, 64] -> [E, N, K/2] (row r's bytes for k = 128c .. 128c+127 are
    block [r//128, c], row r%128); scales [E, NT, KC, 512] -> [E, N, K/32], where the scale of
    (stored row r, block b) is byte (r%32)*16 + ((r%128)//32)*4 + b%4 of group [r//128, b//4].
    """
    E, KC = codes.shape[0], codes.shape[2]
    sr = stored_row_of(N, role)
    # (advanced indices split by a slice put the row axis first: [N, E, KC, 64])
    rows = codes[:, sr // 128, :, sr % 128, :].transpose(1, 0, 2, 3).reshape(E, N, KC * 64)[:, :, : K // 2]
    b = np.arange(K // 32)
    byte = ((sr % 32) * 16 + ((sr % 128) // 32) * 4)[:, None] + (b % 4)[None, :]
    sc = scales[:, (sr // 128)[:, None], (b // 4)[None, :], byte]
    return np.ascontiguousarray(rows), np.ascontiguousarray(sc)


def bf16_dev(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@functools.lru_cache(maxsize=2)
def weights(seed: int, E: int, d: int, I: int, w1_mul: float):
    """GPU MXFP4 weights (library layout) + oracle MXFP4 weights + bit-exactness record."""
    cfg = synth.MoEConfig("w", T=1, d=d, I=I, E=E, k=1, seed=seed, w1_mul=w1_mul)
    dev = "cuda"
    s1c, s1s = moe.mxfp4_shapes(E, 2 * I, d)
    s2c, s2s = moe.mxfp4_shapes(E, d, I)
    g1c = torch.empty(s1c, dtype=torch.uint8, device=dev)
    g1s = torch.empty(s1s, dtype=torch.uint8, device=dev)
    g2c = torch.empty(s2c, dtype=torch.uint8, device=dev)
    g2s = torch.empty(s2s, dtype=torch.uint8, device=dev)
    o1c = np.empty((E, 2 * I, d // 2), np.uint8)
    o1s = np.empty((E, 2 * I, d // 32), np.uint8)
    o2c = np.empty((E, d, I // 2), np.uint8)
    o2s = np.empty((E, d, I // 32), np.uint8)
    mismatches = 0
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for e in range(E):
        for w, gc, gs, oc, os_, role in ((synth.w1_expert(cfg, e), g1c, g1s, o1c, o1s, "gate_up"),
                                         (synth.w2_expert(cfg, e), g2c, g2s, o2c, o2s, "down")):
            wt = torch.from_numpy(w).cuda()
            moe.moe_mxfp4_quantize(wt, gc[e:e + 1], gs[e:e + 1], role=role, status_word=status)
            oc[e], os_[e] = oracle.quantize(w)
            rc, rs = stored_to_rowmajor(gc[e:e + 1].cpu().numpy(), gs[e:e + 1].cpu().numpy(), *w.shape, role)
            mismatches += int(np.count_nonzero(rc[0] != oc[e]))
            mismatches += int(np.count_nonzero(rs[0] != os_[e]))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return dict(gpu=(g1c, g1s, g2c, g2s), oracle=(o1c, o1s, o2c, o2s), mismatches=mismatches)


def case(cfg: synth.MoEConfig):
    """Everything a parity test needs for one workload."""
    x, gamma, rw, rb, attempts, r = routed_inputs(cfg)
    W = weights(cfg.seed, cfg.E, cfg.d, cfg.I, cfg.w1_mul)
    return dict(cfg=cfg, x=x, gamma=gamma, rw=rw, rb=rb, route=r, W=W,
                x_dev=bf16_dev(x), gamma_dev=torch.from_numpy(gamma).cuda(), rw_dev=torch.from_numpy(rw).cuda(),
                rb_dev=torch.from_numpy(rb).cuda())


def run_gpu(c, path, T=None, act="bf16"):
    cfg = c["cfg"]
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path, act=act)
    T = cfg.T
    ws = moe.new_workspace(dims, T)
    y, r = moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws,
                           want_routing=True)
    st = moe.moe_device_status(ws)
    return dict(y=y, routing=r, ws=ws, dims=dims, status=st, act=act)


def oracle_rows(c, tokens=None, want_h=False, act="bf16"):
    cfg = c["cfg"]
    return oracle.moe_forward(c["x"], c["gamma"], c["rw"], c["rb"], *c["W"]["oracle"], I=cfg.I, k=cfg.k,
                              eps=cfg.rms_eps, limit=cfg.swiglu_limit, tokens=tokens, want_h=want_h, act=act)


def parity_stats(y_gpu_u16, y_ref_u16, x_u16) -> dict:
    f = lambda u: synth.bf16_to_f32(u).astype(np.float64)
    yg, yr, x = f(y_gpu_u16), f(y_ref_u16), f(x_u16)
    diff = yg - yr
    rms = float(np.sqrt(np.mean(yr * yr)))
    dref = yr - x
    return dict(rel_fro=float(np.linalg.norm(diff) / np.linalg.norm(yr)),
                max_abs=float(np.abs(diff).max()),
                max_abs_over_rms=float(np.abs(diff).max() / rms),
                delta_rel_fro=float(np.linalg.norm(diff) / max(np.linalg.norm(dref), 1e-30)),
                exact_frac=float(np.mean(y_gpu_u16 == y_ref_u16)))


def assert_parity(st: dict, label: str = "", act: str = "bf16"):
    """The layer's tolerance: relative Frobenius <= 1e-2 and max-abs <= 5e-2 x RMS(y*).

    With MXFP4 activations the element-wise bar is 0.25 x RMS(y*): the GPU forms xe and h
    in fp32 and the oracle in fp64 before the same bf16 rounding and the same E2M1
    quantization, so where a value sits on an E2M1 rounding threshold (or a block's
    largest value on a power of two) the two sides take neighbouring codes.  One such flip
    moves h_i by one E2M1 step, at most half its block's largest value (amax < 8 * 2^s,
    steps up to 2 * 2^s), and y by w * W2[:, i] * dh_i: with |h| blocks up to about 5 and
    |W2| up to about 0.08 at these inputs, up to about 0.2 (0.19 x RMS(y*)).  The
    Frobenius bars, which measure the error over all elements, stay the exact layer's."""
    assert st["rel_fro"] <= 1e-2, (label, st)
    assert st["max_abs_over_rms"] <= (0.25 if act == "mxfp4" else 5e-2), (label, st)
