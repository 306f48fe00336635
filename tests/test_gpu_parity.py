"""GPU parity: the CUDA path through the C ABI against the CPU oracle, same seeded inputs.

Bars: expert indices, per-expert counts, offsets and the grouping bit-exact;
MXFP4 codes and scales bit-exact; outputs within relative Frobenius 1e-2 and
max-abs 5e-2 x RMS(y*) of the oracle.
"""
import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import oracle
import synth
from _gpu_case import (TILE_TOKENS, assert_parity, bf16_dev, bf16_host, case, decode_e2m1_packed, decode_e4m3,
                       oracle_rows, parity_stats, run_gpu, stored_row_of, stored_to_rowmajor, tile_tokens, weights)

pytestmark = pytest.mark.gpu

C = synth.CONFIGS
SMALL = {
    "tiny": C["tiny"],
    "decode_20b": C["decode_20b"],
    "odd": synth.MoEConfig("odd", T=37, d=192, I=320, E=5, k=3),
    "k_eq_E": synth.MoEConfig("k_eq_E", T=24, d=128, I=128, E=4, k=4),
    "single": synth.MoEConfig("single", T=9, d=128, I=192, E=1, k=1),
    "wide_E": synth.MoEConfig("wide_E", T=16, d=256, I=128, E=256, k=8),
    "mid_ragged": synth.MoEConfig("mid_ragged", T=200, d=2880, I=2880, E=8, k=4),
    "clamp": synth.MoEConfig("clamp", T=32, d=2880, I=2880, E=4, k=2, w1_mul=8.0),
    # more than 256 tokens: the tiled router (64- and 32-wide chunks)
    "tiled_route": synth.MoEConfig("tiled_route", T=333, d=256, I=128, E=64, k=4),
    "tiled_wide_E": synth.MoEConfig("tiled_wide_E", T=300, d=256, I=128, E=256, k=8),
}
PATHS = ["gemv", "gemm"]


def _pairs(idx: np.ndarray, perm: np.ndarray, k: int):
    """(token, expert) pairs in sorted order."""
    t = perm // k
    return np.stack([t, idx[t, perm % k]], axis=1)


# ------------------------------------------------------------------------------ quantization


@pytest.mark.parametrize("name", ["tiny", "odd", "decode_20b"])
def test_quantize_bit_exact(name):
    cfg = SMALL[name]
    W = weights(cfg.seed, cfg.E, cfg.d, cfg.I, cfg.w1_mul)
    assert W["mismatches"] == 0


def test_quantize_special_values_bit_exact():
    rng = np.random.default_rng(7)
    rows = []
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.1, 0.2, 0.3, -2.75, 6.0, -7.9, -0.0, 4.0],
                    np.float32)
    rows.append(np.concatenate([ties, ties * -1]))
    rows.append(np.zeros(32, np.float32))                                   # all-zero block
    rows.append(np.full(32, 1e-40, np.float32) * np.arange(32))             # subnormal amax
    rows.append((rng.standard_normal(32) * 3e37).astype(np.float32))        # near the top of fp32
    rows.append(np.exp2(np.arange(-16, 16)).astype(np.float32))             # powers of two
    rows.append(np.nextafter(np.exp2(np.arange(-16, 16)), 0).astype(np.float32))
    w = np.stack(rows).astype(np.float32)
    w = np.concatenate([w, (rng.standard_normal((58, 32)) * 0.02).astype(np.float32)])  # 64 rows
    w = np.tile(w, (1, 2))  # K = 64
    oc, os_ = oracle.quantize(w)
    codes, scales = moe.moe_mxfp4_quantize(torch.from_numpy(w).cuda())
    rc, rs = stored_to_rowmajor(codes.cpu().numpy(), scales.cpu().numpy(), *w.shape, "plain")
    np.testing.assert_array_equal(rc[0], oc)
    np.testing.assert_array_equal(rs[0], os_)
    # the same rows as a gate_up tensor [2I = 128][64]: only the stored row order changes
    w2 = np.concatenate([w, w[::-1]])
    oc2, os2 = oracle.quantize(w2)
    codes, scales = moe.moe_mxfp4_quantize(torch.from_numpy(w2).cuda(), role="gate_up")
    rc, rs = stored_to_rowmajor(codes.cpu().numpy(), scales.cpu().numpy(), *w2.shape, "gate_up")
    np.testing.assert_array_equal(rc[0], oc2)
    np.testing.assert_array_equal(rs[0], os2)


def test_quantize_padding():
    """N = K = 192 pads to 2 x 2 tiles of 128 x 128: padding codes 0, padding scale bytes 127."""
    w = (np.random.default_rng(3).standard_normal((2, 192, 192)) * 0.02).astype(np.float32)
    codes, scales = moe.moe_mxfp4_quantize(torch.from_numpy(w).cuda())
    c, sc = codes.cpu().numpy(), scales.cpu().numpy()
    assert c.shape == (2, 2, 2, 128, 64) and sc.shape == (2, 2, 2, 512)
    assert np.all(c[:, 1, :, 64:, :] == 0)          # rows 192..255
    assert np.all(c[:, :, 1, :, 32:] == 0)          # k 192..255
    sr = stored_row_of(192, "plain")
    mask = np.zeros(sc.shape, bool)
    for b in range(6):
        byte = (sr % 32) * 16 + ((sr % 128) // 32) * 4 + b % 4
        mask[:, sr // 128, b // 4, byte] = True
    assert np.all(sc[~mask] == 127)


def test_quantize_non_finite_is_flagged():
    w = np.ones((64, 64), np.float32)
    w[3, 40] = np.inf
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = moe.moe_mxfp4_quantize(torch.from_numpy(w).cuda(), status_word=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.MOE_ERR_NONFINITE
    _, rs = stored_to_rowmajor(codes.cpu().numpy(), scales.cpu().numpy(), *w.shape, "plain")
    assert rs[0, 3, 1] == 0xFF and rs[0, 3, 0] != 0xFF and rs[0, 2, 1] != 0xFF


# ------------------------------------------------------------------------------ routing / grouping


@pytest.mark.parametrize("name", list(SMALL))
def test_route_bit_exact(name):
    c = case(SMALL[name])
    cfg = c["cfg"]
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k)
    ws = moe.new_workspace(dims, cfg.T)
    out = moe.moe_route(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    idx = out["topk_idx"].cpu().numpy()
    ref = c["route"]
    np.testing.assert_array_equal(np.sort(idx, 1), np.sort(ref["idx"], 1))
    gr = oracle.group(ref["idx"], cfg.E)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), gr["counts"])
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), gr["offsets"])
    np.testing.assert_array_equal(_pairs(idx, out["perm"].cpu().numpy(), cfg.k),
                                  _pairs(ref["idx"], gr["perm"], cfg.k))
    # weights per (token, expert); slot order follows the logits (ties aside)
    wg = out["topk_w"].cpu().numpy()
    for t in range(cfg.T):
        m_g = dict(zip(idx[t].tolist(), wg[t].tolist()))
        m_o = dict(zip(ref["idx"][t].tolist(), ref["w"][t].tolist()))
        for e in m_o:
            assert abs(m_g[e] - m_o[e]) <= 2e-6, (t, e, m_g[e], m_o[e])
    np.testing.assert_allclose(wg.sum(1), 1.0, atol=2e-6)
    lg = ref["logits"][np.arange(cfg.T)[:, None], idx]
    assert np.all(np.diff(lg, axis=1) <= 1e-5)
    # the token tiles: every expert's sorted pairs cut into tiles of the path's size, in
    # expert order (written by the grouping kernel, or by the router's last CTA)
    tt = TILE_TOKENS[moe.resolved_path(dims, cfg.T)]
    want = [(e, int(gr["offsets"][e]) + i * tt, min(tt, int(gr["counts"][e]) - i * tt))
            for e in range(cfg.E) for i in range(-(-int(gr["counts"][e]) // tt))]
    n = int(moe.workspace_view(ws, dims, cfg.T, "ntiles", torch.int32, (1,)).item())
    assert n == len(want)
    got = moe.workspace_view(ws, dims, cfg.T, "tiles", torch.int32, (n, 4)).cpu().numpy()[:, :3]
    np.testing.assert_array_equal(got, np.array(want, dtype=np.int32).reshape(-1, 3))


# ------------------------------------------------------------------------------ whole layer


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_parity(name, path):
    c = case(SMALL[name])
    cfg = c["cfg"]
    g = run_gpu(c, path)
    assert g["status"] == moe.MOE_OK, moe.status_string(g["status"])
    ref = oracle_rows(c)
    st = parity_stats(bf16_host(g["y"]), ref["y"], c["x"])
    assert_parity(st, f"{name}/{path}")
    assert st["delta_rel_fro"] <= 2.5e-2, st
    np.testing.assert_array_equal(np.sort(g["routing"]["topk_idx"].cpu().numpy(), 1), np.sort(ref["idx"], 1))


def _h_from_workspace_fp4(g, cfg):
    """h [P, I] from the down GEMM's packed MXFP4 blocks: per token tile and 128-chunk, one
    row of 64 bytes per token (16-byte unit u of row n stored at unit u ^ ((n // 2) % 4);
    element 2i in the low nibble of byte i), then the scale-factor groups."""
    dims, ws, T = g["dims"], g["ws"], cfg.T
    P = T * cfg.k
    KC = moe.kpad128(cfg.I) // 128
    bt = tile_tokens(moe.resolved_path(dims, T), "mxfp4")
    G = (bt + 127) // 128
    BB = (bt * 64 + G * 512 + 1023) // 1024 * 1024
    view = lambda f, dt, sh: moe.workspace_view(ws, dims, T, f, dt, sh).cpu().numpy()
    offsets = view("offsets", torch.int32, (cfg.E + 1,))
    tbase = view("tile_base", torch.int32, (cfg.E,))
    n_tiles = (P + bt - 1) // bt + cfg.E
    bph = view("bph", torch.uint8, (n_tiles, KC, BB))
    h = np.empty((P, cfg.I))
    b = np.arange(cfg.I // 32)
    u = np.arange(4)
    for p in range(P):
        e = int(np.searchsorted(offsets, p, side="right") - 1)
        j = p - offsets[e]
        tile, n = tbase[e] + j // bt, j % bt
        phys = n * 64 + ((u ^ ((n >> 1) % 4)) << 4)
        rows = bph[tile][:, (phys[:, None] + np.arange(16)[None, :]).ravel()]      # [KC, 64]
        vals = decode_e2m1_packed(rows).reshape(-1)[: cfg.I]
        sfo = bt * 64 + (n // 128) * 512 + (n % 32) * 16 + ((n % 128) // 32) * 4 + b % 4
        sc = bph[tile, b // 4, sfo].astype(np.float64) - 127
        h[p] = vals * np.repeat(np.exp2(sc), 32)
    return h


def _h_from_workspace(g, cfg):
    """h [P, I] (sorted pairs) rebuilt from the down GEMM's packed activation blocks: per
    token tile and 128-chunk, terms*BN E4M3 rows (row n = term n % terms of token
    n // terms: hi / lo for bf16 activations, one row for MXFP8; 16-byte unit u stored at
    unit u ^ (n % 8)), then the scale-factor groups (byte (n%32)*16 + ((n%128)//32)*4 + b%4
    of group n // 128 for 32-block b)."""
    dims, ws, T = g["dims"], g["ws"], cfg.T
    P = T * cfg.k
    Ip = moe.kpad128(cfg.I)
    KC = Ip // 128
    nterms = 1 if g["act"] == "mxfp8" else 2
    bt = tile_tokens(moe.resolved_path(dims, T), g["act"])
    R = nterms * bt
    G = (R + 127) // 128
    BB = (R * 128 + G * 512 + 1023) // 1024 * 1024
    view = lambda f, dt, sh: moe.workspace_view(ws, dims, T, f, dt, sh).cpu().numpy()
    offsets = view("offsets", torch.int32, (cfg.E + 1,))
    tbase = view("tile_base", torch.int32, (cfg.E,))
    n_tiles = (P + bt - 1) // bt + cfg.E
    bph = view("bph", torch.uint8, (n_tiles, KC, BB))
    h = np.empty((P, cfg.I))
    b = np.arange(cfg.I // 32)
    u = np.arange(8)
    for p in range(P):
        e = int(np.searchsorted(offsets, p, side="right") - 1)
        j = p - offsets[e]
        tile, col = tbase[e] + j // bt, j % bt
        terms = []
        for n in range(nterms * col, nterms * col + nterms):
            phys = n * 128 + ((u ^ (n % 8)) << 4)                                    # [8]
            rows = bph[tile][:, (phys[:, None] + np.arange(16)[None, :]).ravel()]     # [KC, 128]
            codes = rows.reshape(-1)[: cfg.I]
            sfo = R * 128 + (n // 128) * 512 + (n % 32) * 16 + ((n % 128) // 32) * 4 + b % 4
            sc = bph[tile, b // 4, sfo].astype(np.float64) - 127
            terms.append(decode_e4m3(codes) * np.repeat(np.exp2(sc), 32))
        h[p] = sum(terms)
    return h


@pytest.mark.parametrize("path", PATHS)
def test_swiglu_output_h_matches_oracle(path):
    """The gate_up stage alone: h rebuilt from its E4M3 hi / lo terms vs the oracle's h;
    the two terms carry bf16 values exactly (up to the block's dynamic range)."""
    c = case(SMALL["mid_ragged"])
    cfg = c["cfg"]
    g = run_gpu(c, path)
    assert g["status"] == moe.MOE_OK
    P = cfg.T * cfg.k
    h = _h_from_workspace(g, cfg)
    inv = moe.workspace_view(g["ws"], g["dims"], cfg.T, "inv", torch.int32, (P,)).cpu().numpy()
    idx = g["routing"]["topk_idx"].cpu().numpy()
    ref = oracle_rows(c, want_h=True)
    href = synth.bf16_to_f32(ref["h"]).astype(np.float64)  # [T, k, I] in the oracle's slot order
    num = den = 0.0
    for t in range(cfg.T):
        for s in range(cfg.k):
            so = int(np.nonzero(ref["idx"][t] == idx[t, s])[0][0])
            diff = h[inv[t * cfg.k + s]] - href[t, so]
            num += float(diff @ diff)
            den += float(href[t, so] @ href[t, so])
    assert np.sqrt(num / den) <= 1e-2
    # hi + lo reproduce bf16 values: round-tripping through bf16 changes (almost) nothing
    h32 = h.astype(np.float32)
    u = h32.view(np.uint32).astype(np.uint64)
    hb = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)
    assert np.mean(hb == h32) >= 0.999, np.mean(hb == h32)


# ------------------------------------------------------------------------------ MXFP8 activations
# MOE_ACT_MXFP8: the expert inputs and the SwiGLU outputs quantized to E4M3 in 32-value
# blocks; the oracle models the same quantization (act="mxfp8").  Same bars as the bf16
# format, plus the distance to the exact-bf16 layer, which the format is allowed to move.


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_parity_mxfp8(name, path):
    c = case(SMALL[name])
    cfg = c["cfg"]
    g = run_gpu(c, path, act="mxfp8")
    assert g["status"] == moe.MOE_OK, moe.status_string(g["status"])
    ref = oracle_rows(c, act="mxfp8")
    y = bf16_host(g["y"])
    st = parity_stats(y, ref["y"], c["x"])
    assert_parity(st, f"{name}/{path}/mxfp8")
    assert st["delta_rel_fro"] <= 2.5e-2, st
    np.testing.assert_array_equal(np.sort(g["routing"]["topk_idx"].cpu().numpy(), 1), np.sort(ref["idx"], 1))
    # What the format itself costs against the exact layer (bf16 activations), on the
    # oracle's unrounded outputs: it moves the expert output y - x by a few percent of its
    # norm (about 5% at d = I = 2880; not within the exact layer's tolerance on y there).
    x = synth.bf16_to_f32(c["x"]).astype(np.float64)
    y_bf = oracle_rows(c)["y_f64"]
    moved = np.linalg.norm(ref["y_f64"] - y_bf) / np.linalg.norm(y_bf - x)
    assert 1e-3 < moved < 0.1, moved


@pytest.mark.parametrize("path", PATHS)
def test_swiglu_output_h_mxfp8(path):
    """h as the down GEMM reads it with MXFP8 activations: one E4M3 row per token with its
    block scale, equal to the oracle's quantized h up to rare one-step rounding flips (h is
    computed in fp32 here and in fp64 there before both round it)."""
    c = case(SMALL["mid_ragged"])
    cfg = c["cfg"]
    g = run_gpu(c, path, act="mxfp8")
    assert g["status"] == moe.MOE_OK
    P = cfg.T * cfg.k
    h = _h_from_workspace(g, cfg)
    inv = moe.workspace_view(g["ws"], g["dims"], cfg.T, "inv", torch.int32, (P,)).cpu().numpy()
    idx = g["routing"]["topk_idx"].cpu().numpy()
    ref = oracle_rows(c, want_h=True, act="mxfp8")
    href = synth.bf16_to_f32(ref["h"]).astype(np.float64)
    same = total = 0
    num = den = 0.0
    for t in range(cfg.T):
        for s in range(cfg.k):
            so = int(np.nonzero(ref["idx"][t] == idx[t, s])[0][0])
            a, b = h[inv[t * cfg.k + s]], href[t, so]
            same += int(np.count_nonzero(a == b))
            total += a.size
            num += float((a - b) @ (a - b))
            den += float(b @ b)
    assert same / total >= 0.99, same / total
    assert np.sqrt(num / den) <= 1e-2


# ------------------------------------------------------------------------------ MXFP4 activations
# MOE_ACT_MXFP4: the expert inputs and the SwiGLU outputs quantized with the weights' own
# format (E2M1 in 32-value blocks); the FP4 x FP4 MMA.  The oracle models the same
# quantization (act="mxfp4").  Same bars as the other formats, against that oracle.


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_parity_mxfp4(name, path):
    c = case(SMALL[name])
    g = run_gpu(c, path, act="mxfp4")
    assert g["status"] == moe.MOE_OK, moe.status_string(g["status"])
    ref = oracle_rows(c, act="mxfp4")
    st = parity_stats(bf16_host(g["y"]), ref["y"], c["x"])
    assert_parity(st, f"{name}/{path}/mxfp4", "mxfp4")
    assert st["delta_rel_fro"] <= 2.5e-2, st
    np.testing.assert_array_equal(np.sort(g["routing"]["topk_idx"].cpu().numpy(), 1), np.sort(ref["idx"], 1))


@pytest.mark.parametrize("path", PATHS)
def test_swiglu_output_h_mxfp4(path):
    """h as the down GEMM reads it with MXFP4 activations: one row of packed E2M1 codes per
    token with its block scales, equal to the oracle's quantized h up to rare one-step
    rounding flips (h is computed in fp32 here and in fp64 there before both round it)."""
    c = case(SMALL["mid_ragged"])
    cfg = c["cfg"]
    g = run_gpu(c, path, act="mxfp4")
    assert g["status"] == moe.MOE_OK
    P = cfg.T * cfg.k
    h = _h_from_workspace_fp4(g, cfg)
    inv = moe.workspace_view(g["ws"], g["dims"], cfg.T, "inv", torch.int32, (P,)).cpu().numpy()
    idx = g["routing"]["topk_idx"].cpu().numpy()
    ref = oracle_rows(c, want_h=True, act="mxfp4")
    href = synth.bf16_to_f32(ref["h"]).astype(np.float64)
    same = total = 0
    num = den = 0.0
    for t in range(cfg.T):
        for s in range(cfg.k):
            so = int(np.nonzero(ref["idx"][t] == idx[t, s])[0][0])
            a, b = h[inv[t * cfg.k + s]], href[t, so]
            same += int(np.count_nonzero(a == b))
            total += a.size
            num += float((a - b) @ (a - b))
            den += float(b @ b)
    assert same / total >= 0.99, same / total
    assert np.sqrt(num / den) <= 1e-2


# ------------------------------------------------------------------------------ edge cases


def test_T_zero_and_one():
    c = case(SMALL["tiny"])
    cfg = c["cfg"]
    for path in PATHS:
        dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, path=path)
        ws = moe.new_workspace(dims, 1)
        y = moe.moe_forward(dims, c["x_dev"][:1], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
        assert moe.moe_device_status(ws) == moe.MOE_OK
        ref = oracle_rows(c, tokens=np.array([0], np.int32))
        assert_parity(parity_stats(bf16_host(y), ref["y"], c["x"][:1]), path)
        # T = 0 launches nothing
        moe.moe_forward(dims, c["x_dev"][:0], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
        assert moe.last_launch_count() == 0


def test_deterministic():
    c = case(SMALL["mid_ragged"])
    for path in ("gemm", "gemv"):
        a = bf16_host(run_gpu(c, path)["y"])
        b = bf16_host(run_gpu(c, path)["y"])
        np.testing.assert_array_equal(a, b)


def _set_scale(scales_gpu, scales_or, e, n, b, value, N, K, role):
    """Set the E8M0 scale of (expert e, logical row n, block b) on both sides."""
    sr = int(stored_row_of(N, role)[n])
    byte = (sr % 32) * 16 + ((sr % 128) // 32) * 4 + b % 4
    scales_gpu[e, sr // 128, b // 4, byte] = value
    scales_or[e, n, b] = value


@pytest.mark.parametrize("path", PATHS)
def test_extreme_scales_stay_exact(path):
    """The tensor cores apply E8M0 scales exactly over their whole range: blocks scaled by
    2^+-40 (far outside f16) still match the oracle."""
    c = case(SMALL["tiny"])
    cfg = c["cfg"]
    g1c, g1s, g2c, g2s = (t.clone() for t in c["W"]["gpu"])
    o1c, o1s, o2c, o2s = (a.copy() for a in c["W"]["oracle"])
    rng = np.random.default_rng(11)
    for _ in range(6):
        e, n, b = int(rng.integers(cfg.E)), int(rng.integers(2 * cfg.I)), int(rng.integers(cfg.d // 32))
        _set_scale(g1s, o1s, e, n, b, int(o1s[e, n, b]) + 40, 2 * cfg.I, cfg.d, "gate_up")  # g / u saturate
        e, n, b = int(rng.integers(cfg.E)), int(rng.integers(cfg.d)), int(rng.integers(cfg.I // 32))
        _set_scale(g2s, o2s, e, n, b, int(o2s[e, n, b]) - 40, cfg.d, cfg.I, "down")
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, path=path)
    ws = moe.new_workspace(dims, cfg.T)
    y = moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], g1c, g1s, g2c, g2s, ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    ref = oracle.moe_forward(c["x"], c["gamma"], c["rw"], c["rb"], o1c, o1s, o2c, o2s, I=cfg.I, k=cfg.k,
                             eps=cfg.rms_eps, limit=cfg.swiglu_limit)
    assert_parity(parity_stats(bf16_host(y), ref["y"], c["x"]), path)


def test_non_finite_input_is_reported():
    c = case(SMALL["tiny"])
    cfg = c["cfg"]
    x = c["x"].copy()
    x[3, 5] = 0x7F80  # +inf
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, path="gemm")
    ws = moe.new_workspace(dims, cfg.T)
    moe.moe_forward(dims, bf16_dev(x), c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
    assert moe.moe_device_status(ws) == moe.MOE_ERR_NONFINITE
    assert moe.moe_device_status(ws) == moe.MOE_OK  # reading clears the word


def test_launch_count_reported():
    c = case(SMALL["tiny"])
    cfg = c["cfg"]
    for path, n in (("gemm", 6),   # route, group, pack, gate_up, down, combine
                    ("gemv", 5)):  # route (+ grouping), pack, gate_up, down, combine
        dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, path=path)
        ws = moe.new_workspace(dims, cfg.T)
        moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
        assert moe.last_launch_count() == n, path
