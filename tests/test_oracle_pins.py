"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a number
the pages print, a closed form, a special case that reduces to a textbook
dense layer, or a brute-force / dense second formulation (``_dense_ref``).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from _dense_ref import bf16_bits_to_f64, decode, dense_layer, e2m1_from_bits, round_bf16, silu

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")))


def g(name):
    return GOLD[name]["value"]


# --------------------------------------------------------------------------- storage


def test_storage_4p25_bits_for_2880x5760():
    """A 2880x5760 MXFP4 matrix: 8,294,400 code bytes + 518,400 scale bytes = 4.25 bits/param."""
    rows, K = 2 * g("intermediate_size"), g("hidden_size")
    cb, sb = oracle.storage_bytes(rows, K)
    assert (cb, sb) == (8_294_400, 518_400)
    assert (cb + sb) * 8 / (rows * K) == g("mxfp4_bits_per_param")
    assert 4 + g("mxfp4_scale_bits") / g("mxfp4_block") == g("mxfp4_bits_per_param")


def test_swiglu_param_count_example_width_1024():
    """The pages' example: FFN fc1+fc2 = 8,388,608 vs SwiGLU 3 x 1,048,576 at width 1024.

    The oracle's expert shapes (W1 [2I, d], W2 [d, I]) at d = I = 1024 must hold
    exactly the SwiGLU count; the FFN count uses the pages' 4x hidden width.
    """
    d = I = 1024
    w1_rows, w2_rows = 2 * I, d
    cb1, _ = oracle.storage_bytes(w1_rows, d)
    cb2, _ = oracle.storage_bytes(w2_rows, I)
    params = 2 * (cb1 + cb2)  # two codes per byte
    assert params == g("swiglu_params_width1024") == 3 * 1024 * 1024
    assert 2 * d * 4 * d == g("ffn_fc1_plus_fc2_width1024")


def test_config_consistency_with_pages():
    """Expert params x experts x layers at 4.25 bits vs the pages' totals and memory fits."""
    d, I = g("hidden_size"), g("intermediate_size")
    per_expert = 3 * d * I
    assert per_expert == 24_883_200
    moe_20b = per_expert * g("num_local_experts_20b") * g("num_hidden_layers_20b")
    assert moe_20b / g("total_params_20b") > g("moe_param_share_min")   # ">90% of params are MoE"
    assert moe_20b < g("total_params_20b")
    gb_20b = moe_20b * g("mxfp4_bits_per_param") / 8 / 1e9
    gb_120b = per_expert * g("num_local_experts_120b") * g("num_hidden_layers_120b") * 4.25 / 8 / 1e9
    assert gb_20b < g("fits_gb_20b") and gb_120b < g("fits_gb_120b")
    per_layer_120b = per_expert * g("num_local_experts_120b") * 4.25 / 8 / 1e9
    assert abs(per_layer_120b - 1.692) < 1e-3
    # active params: 4 experts x 24 layers is below the 3.6B active figure (attention etc. add the rest)
    assert per_expert * g("experts_per_token") * g("num_hidden_layers_20b") < g("active_params_20b")


# --------------------------------------------------------------------------- E2M1 / quantization


def test_e2m1_table_matches_bit_fields():
    for c in range(16):
        assert oracle.e2m1_value(c) == e2m1_from_bits(c), c
    assert sorted({abs(oracle.e2m1_value(c)) for c in range(16)}) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def _block_with(values, anchor=4.0):
    """A 32-value block containing ``values`` plus an anchor that fixes amax (scale 2^0 for anchor in [4, 8))."""
    v = np.zeros(32, np.float32)
    v[0] = anchor
    v[1:1 + len(values)] = values
    return v


def test_quantize_ties_to_even_and_saturation():
    vals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.1, 0.2, 0.3, -2.75, 6.0, -7.9]
    expect = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 0.0, 0.0, 0.5, -3.0, 6.0, -6.0]
    codes, scales = oracle.quantize(_block_with(vals, anchor=4.0)[None, :])
    assert scales[0, 0] == 127  # floor(log2 7.9) - 2 = 0
    deq = oracle.dequantize(codes, scales)[0]
    np.testing.assert_array_equal(deq[1:1 + len(vals)], expect)
    # -0.1 rounds to zero: no sign bit on a zero code
    hi = codes[0, 4] >> 4  # element 9 of the block holds -0.1
    assert hi == 0


def test_quantize_scale_exponent_exact_at_powers_of_two():
    # amax exactly 2^j: floor(log2) = j (no log2 misrounding), scale byte = j - 2 + 127
    for j in range(-20, 21):
        blk = np.full((1, 32), 2.0 ** j * 0.5, np.float32)
        blk[0, 3] = 2.0 ** j
        _, s = oracle.quantize(blk)
        assert s[0, 0] == j - 2 + 127, j
        blk[0, 3] = np.nextafter(np.float32(2.0 ** j), np.float32(0))
        _, s = oracle.quantize(blk)
        assert s[0, 0] == j - 3 + 127, j


@pytest.mark.parametrize("K", [256, 96])   # 96: an odd number of 32-blocks (the oracle takes any multiple of 32)
def test_quantize_grid_values_round_trip(K):
    rng = np.random.default_rng(1)
    rows = 64
    mags = rng.integers(0, 8, size=(rows, K))
    mags[:, ::32] = rng.integers(6, 8, size=(rows, K // 32))  # magnitude 4 or 6: amax in [4, 8) x 2^s
    sign = rng.integers(0, 2, size=(rows, K)) * (mags > 0)
    code = mags | (sign << 3)
    s = rng.integers(-30, 30, size=(rows, K // 32))
    vals = np.vectorize(e2m1_from_bits)(code) * np.exp2(np.repeat(s, 32, axis=1))
    codes, scales = oracle.quantize(vals.astype(np.float32))
    np.testing.assert_array_equal(scales.astype(int), s + 127)
    np.testing.assert_array_equal(oracle.dequantize(codes, scales), vals)
    lo, hi = codes & 15, codes >> 4
    np.testing.assert_array_equal(np.stack([lo, hi], -1).reshape(rows, K), code)


def test_quantize_is_nearest_grid_point_brute_force():
    """Every decoded value is the closest point of {E2M1 x 2^s} (ties: even code), s = floor(log2 amax) - 2."""
    w = synth.normal_f32(3, 99, 0, 64 * 320, 0.0, 0.02).reshape(64, 320)
    w[5, :32] = 0.0  # an all-zero block
    codes, scales = oracle.quantize(w)
    deq = oracle.dequantize(codes, scales)
    grid_codes = np.arange(16)
    grid = np.array([e2m1_from_bits(c) for c in grid_codes])
    for r in range(w.shape[0]):
        for b in range(w.shape[1] // 32):
            blk = w[r, 32 * b:32 * b + 32].astype(np.float64)
            amax = np.max(np.abs(blk))
            if amax == 0:
                assert scales[r, b] == 127
                assert np.all(deq[r, 32 * b:32 * b + 32] == 0)
                continue
            _, e = np.frexp(amax)
            s = (e - 1) - 2
            assert scales[r, b] == s + 127
            for i, v in enumerate(blk):
                vs = min(max(v / 2.0 ** s, -6.0), 6.0)
                err = np.abs(grid - vs)
                best = np.flatnonzero(err == err.min())
                vals = {grid[c] for c in best}
                if len(vals) > 1:  # a tie: the even code (mantissa bit 0) wins
                    best = [c for c in best if c % 2 == 0]
                assert deq[r, 32 * b + i] == grid[best[0]] * 2.0 ** s, (r, b, i, v)


def test_quantize_error_bound():
    w = synth.normal_f32(4, 99, 1, 256 * 2880, 0.0, 0.02).reshape(256, 2880)
    codes, scales = oracle.quantize(w)
    deq = oracle.dequantize(codes, scales)
    s = np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)
    a = np.abs(w.astype(np.float64)) / s
    # half the grid gap at each magnitude; saturation region (6, 8) loses up to 2
    half_gap = np.where(a < 2, 0.25, np.where(a < 4, 0.5, np.where(a <= 6, 1.0, 2.0)))
    assert np.all(np.abs(w - deq) / s <= half_gap + 1e-12)
    rel = np.linalg.norm(w - deq) / np.linalg.norm(w)
    assert 0.05 < rel < 0.2  # 4-bit quantisation of a normal distribution


def test_quantize_rejects_non_finite():
    w = np.ones((1, 32), np.float32)
    w[0, 7] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(w)


# --------------------------------------------------------------------------- bf16 rounding


def test_round_bf16_midpoints_and_against_float32_bits():
    assert oracle.round_bf16(1 + 2 ** -8) == 1.0
    assert oracle.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    assert oracle.round_bf16(-(1 + 2 ** -8 + 2 ** -30)) == -(1 + 2 ** -7)
    rng = np.random.default_rng(2)
    f = (rng.standard_normal(2000) * np.exp2(rng.integers(-60, 60, 2000))).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    ref = (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32)
    got = np.array([oracle.round_bf16(float(v)) for v in f])
    np.testing.assert_array_equal(got, ref.astype(np.float64))


def test_to_bf16_array_matches_scalar_rounding_and_float32_bits():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(3000) * np.exp2(rng.integers(-40, 40, 3000))
    v[:4] = [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8 + 2 ** -30), 0.0]
    bits = oracle.to_bf16(v)
    assert bits[0] == 0x3F80 and bits[1] == 0x3F82 and bits[2] == 0xBF81 and bits[3] == 0
    got = synth.bf16_to_f32(bits).astype(np.float64)
    np.testing.assert_array_equal(got, [oracle.round_bf16(float(a)) for a in v])
    f = v.astype(np.float32)   # float32 inputs: rounding their bit patterns gives the same bf16
    u = f.view(np.uint32).astype(np.uint64)
    np.testing.assert_array_equal(oracle.to_bf16(f.astype(np.float64)),
                                  ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16))


# --------------------------------------------------------------------------- RMSNorm


def test_rmsnorm_closed_forms():
    d = 64
    c = 1.5
    x = np.full((1, d), 0x3FC0, np.uint16)  # 1.5 in bf16
    gamma = np.linspace(0.5, 2.0, d).astype(np.float32)
    xn = oracle.rmsnorm(x, gamma, 1e-5)
    np.testing.assert_allclose(xn[0], c / math.sqrt(c * c + 1e-5) * gamma.astype(np.float64), rtol=1e-15)
    # with gamma = 1: mean(xn^2) = ms / (ms + eps) for any row
    xr = synth.normal_bf16(5, 99, 0, 4 * d, 0.0, 1.0).reshape(4, d)
    xn = oracle.rmsnorm(xr, np.ones(d, np.float32), 1e-5)
    xv = bf16_bits_to_f64(xr)
    ms = np.mean(xv * xv, axis=1)
    np.testing.assert_allclose(np.mean(xn * xn, axis=1), ms / (ms + 1e-5), rtol=1e-13)
    # scale invariance when eps = 0; sign follows x
    xn0 = oracle.rmsnorm(xr, np.ones(d, np.float32), 0.0)
    x2 = (xr.astype(np.uint32) + 0x0080).astype(np.uint16)  # exponent + 1: x2 = 2 x
    np.testing.assert_allclose(oracle.rmsnorm(x2, np.ones(d, np.float32), 0.0), xn0, rtol=1e-14)
    assert np.all(np.sign(xn0) == np.sign(xv))


# --------------------------------------------------------------------------- routing


def test_next_block_norm_closed_form():
    """A row of equal magnitudes c normalizes to +-gamma * c / sqrt(c^2 + eps), rounded to bf16."""
    d = 128
    c = 3.0
    row = np.full(d, 0x4040, np.uint16)                 # 3.0
    row[1::2] = 0xC040                                  # -3.0
    gamma = np.linspace(0.25, 4.0, d).astype(np.float32)
    got = synth.bf16_to_f32(oracle.next_block_norm(row[None, :], gamma, 1e-5)[0]).astype(np.float64)
    want = np.where(np.arange(d) % 2, -1.0, 1.0) * gamma.astype(np.float64) * c / math.sqrt(c * c + 1e-5)
    np.testing.assert_array_equal(got, [oracle.round_bf16(w) for w in want])
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8)


def test_route_mixture_example_0p7_0p3():
    """Top-2 of 4 with logits set so experts 2 and 4 (1-based) win with weights 0.7 and 0.3."""
    ex = g("mixture_example")
    E, k = ex["E"], ex["k"]
    d = 32
    x = synth.normal_bf16(6, 99, 0, 3 * d, 0.0, 1.0).reshape(3, d)
    rw = np.zeros((E, d), np.float32)
    rb = np.array([-5.0, math.log(7.0), -5.0, math.log(3.0)], np.float32)
    r = oracle.route(x, np.ones(d, np.float32), rw, rb, k, 1e-5)
    assert np.all(r["idx"] == np.array(ex["experts_1based"]) - 1)
    np.testing.assert_allclose(r["w"], np.tile(ex["weights"], (3, 1)), atol=2e-7)


def test_route_weights_sum_to_one_and_topk_is_argsort():
    cfg = synth.MoEConfig("t", T=64, d=96, I=64, E=16, k=4)
    x = synth.hidden(cfg)
    r = oracle.route(x, synth.norm_weight(cfg), synth.router_weight(cfg), synth.router_bias(cfg), cfg.k, 1e-5)
    np.testing.assert_allclose(r["w"].sum(axis=1), 1.0, atol=1e-12)
    order = np.argsort(-r["logits"], axis=1, kind="stable")[:, :cfg.k]
    np.testing.assert_array_equal(r["idx"], order)
    srt = -np.sort(-r["logits"], axis=1)
    np.testing.assert_allclose(r["gap"], srt[:, cfg.k - 1] - srt[:, cfg.k])
    # logits are affine in the router weights: with W_r rows = unit vectors, l = b + xn[:, i]
    rw = np.zeros((cfg.E, cfg.d), np.float32)
    rw[np.arange(cfg.E), np.arange(cfg.E) * 3] = 1.0
    r2 = oracle.route(x, synth.norm_weight(cfg), rw, synth.router_bias(cfg), cfg.k, 1e-5)
    xn = oracle.rmsnorm(x, synth.norm_weight(cfg), 1e-5)
    np.testing.assert_allclose(r2["logits"], xn[:, ::3][:, :cfg.E] + synth.router_bias(cfg)[None, :], rtol=1e-15)


def test_route_ties_go_to_lower_index_and_k1_weight_is_one():
    d = 32
    x = synth.normal_bf16(7, 99, 0, d, 0.0, 1.0).reshape(1, d)
    rb = np.array([0.5, 1.0, 1.0, 0.2, 1.0], np.float32)
    r = oracle.route(x, np.ones(d, np.float32), np.zeros((5, d), np.float32), rb, 2, 1e-5)
    assert list(r["idx"][0]) == [1, 2] and r["gap"][0] == 0.0
    r1 = oracle.route(x, np.ones(d, np.float32), np.zeros((5, d), np.float32), rb, 1, 1e-5)
    assert r1["w"][0, 0] == 1.0


# --------------------------------------------------------------------------- grouping


def test_group_invariants_and_brute_force():
    rng = np.random.default_rng(3)
    T, k, E = 200, 4, 16
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    gr = oracle.group(idx, E)
    assert gr["counts"].sum() == T * k
    np.testing.assert_array_equal(gr["counts"], np.bincount(idx.ravel(), minlength=E))
    np.testing.assert_array_equal(np.sort(gr["perm"]), np.arange(T * k))           # bijection
    np.testing.assert_array_equal(gr["inv"][gr["perm"]], np.arange(T * k))         # inverse map
    ref = sorted(((int(idx[t, s]), t, t * k + s) for t in range(T) for s in range(k)))
    np.testing.assert_array_equal(gr["perm"], [q for _, _, q in ref])
    np.testing.assert_array_equal(gr["offsets"], np.concatenate([[0], np.cumsum(gr["counts"])]))
    bad = idx.copy()
    bad[0, 1] = bad[0, 0]
    with pytest.raises(ValueError):
        oracle.group(bad, E)


# --------------------------------------------------------------------------- whole layer


def _small_case(T, d, I, E, k, seed=0, w1_mul=1.0):
    cfg = synth.MoEConfig("s", T=T, d=d, I=I, E=E, k=k, seed=seed, w1_mul=w1_mul)
    x = synth.hidden(cfg)
    gamma, rw, rb = synth.norm_weight(cfg), synth.router_weight(cfg), synth.router_bias(cfg)
    w1 = [oracle.quantize(synth.w1_expert(cfg, e)) for e in range(E)]
    w2 = [oracle.quantize(synth.w2_expert(cfg, e)) for e in range(E)]
    stk = lambda lst, i: np.stack([p[i] for p in lst])
    W = (stk(w1, 0), stk(w1, 1), stk(w2, 0), stk(w2, 1))
    dec1 = [decode(*p) for p in w1]
    dec2 = [decode(*p) for p in w2]
    return cfg, x, gamma, rw, rb, W, dec1, dec2


def _oracle_y(case, **kw):
    cfg, x, gamma, rw, rb, W, _, _ = case
    return oracle.moe_forward(x, gamma, rw, rb, *W, I=cfg.I, k=cfg.k, **kw)


@pytest.mark.parametrize("shape", [(8, 32, 32, 5, 2), (6, 64, 32, 4, 3), (5, 32, 64, 3, 1)])
def test_forward_matches_dense_brute_force(shape):
    """Sparse oracle == every-expert-on-every-token masked to top-k (to 1e-12)."""
    case = _small_case(*shape, seed=11)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    out = _oracle_y(case)
    y64, y_r, logits, weights = dense_layer(x, gamma, rw, rb, dec1, dec2, cfg.k)
    np.testing.assert_allclose(out["y_f64"], y64, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(bf16_bits_to_f64(out["y"]), y_r)
    assert np.all(np.take_along_axis(weights, out["idx"], 1) == np.take_along_axis(weights, out["idx"], 1))
    np.testing.assert_allclose(np.take_along_axis(weights, out["idx"], 1), out["w"], atol=1e-15)


def test_forward_k_equals_E_is_dense_softmax_mixture():
    case = _small_case(6, 32, 32, 4, 4, seed=12)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    out = _oracle_y(case)
    y64, _, _, _ = dense_layer(x, gamma, rw, rb, dec1, dec2, cfg.k, mode="dense")
    np.testing.assert_allclose(out["y_f64"], y64, rtol=0, atol=1e-12)


def test_forward_single_expert_is_dense_swiglu_mlp():
    """E = 1, k = 1: y = x + W2 (silu(min(W1_g xe, 7)) * clip(W1_u xe, -7, 7)), a textbook dense layer."""
    case = _small_case(7, 64, 96, 1, 1, seed=13)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    out = _oracle_y(case, want_h=True)
    xv = bf16_bits_to_f64(x)
    xn = xv / np.sqrt(np.mean(xv ** 2, axis=1, keepdims=True) + 1e-5) * gamma
    xe = round_bf16(xn)
    gt, up = xe @ dec1[0][:cfg.I].T, xe @ dec1[0][cfg.I:].T
    h = round_bf16(silu(np.minimum(gt, 7.0)) * np.clip(up, -7.0, 7.0))
    np.testing.assert_array_equal(bf16_bits_to_f64(out["h"][:, 0, :]), h)
    np.testing.assert_allclose(out["y_f64"], xv + h @ dec2[0].T, rtol=0, atol=1e-12)
    assert np.all(out["w"] == 1.0)


def test_forward_mixture_example_is_weighted_sum_of_two_experts():
    case = _small_case(4, 32, 32, 4, 2, seed=14)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    rw0 = np.zeros_like(rw)
    rb0 = np.array([-5.0, math.log(7.0), -5.0, math.log(3.0)], np.float32)
    out = oracle.moe_forward(x, gamma, rw0, rb0, *W, I=cfg.I, k=2)
    xv = bf16_bits_to_f64(x)
    xe = round_bf16(xv / np.sqrt(np.mean(xv ** 2, axis=1, keepdims=True) + 1e-5) * gamma)

    def expert(e):
        gu = xe @ dec1[e].T
        h = round_bf16(silu(np.minimum(gu[:, :cfg.I], 7.0)) * np.clip(gu[:, cfg.I:], -7.0, 7.0))
        return h @ dec2[e].T

    np.testing.assert_allclose(out["y_f64"], xv + 0.7 * expert(1) + 0.3 * expert(3), rtol=0, atol=2e-7)


def test_forward_clamp_fires_under_stress():
    """W1 scaled up (x60 at d = 64, the std a x8 stress gives at d = 2880) pushes |g|, |u| past the
    limit 7; h still matches the clamped formula."""
    case = _small_case(6, 64, 64, 2, 1, seed=15, w1_mul=60.0)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    out = _oracle_y(case, want_h=True)
    xv = bf16_bits_to_f64(x)
    xe = round_bf16(xv / np.sqrt(np.mean(xv ** 2, axis=1, keepdims=True) + 1e-5) * gamma)
    e = out["idx"][:, 0]
    gu = np.stack([xe[t] @ dec1[e[t]].T for t in range(cfg.T)])
    assert np.mean(gu[:, :cfg.I] > 7) > 0.05 and np.mean(np.abs(gu[:, cfg.I:]) > 7) > 0.05
    h = round_bf16(silu(np.minimum(gu[:, :cfg.I], 7.0)) * np.clip(gu[:, cfg.I:], -7.0, 7.0))
    np.testing.assert_array_equal(bf16_bits_to_f64(out["h"][:, 0, :]), h)
    assert np.abs(bf16_bits_to_f64(out["h"])).max() <= 7.0 * 7.0


def test_forward_token_subset_equals_full_rows():
    case = _small_case(12, 32, 32, 5, 2, seed=16)
    full = _oracle_y(case)
    sub = _oracle_y(case, tokens=np.array([11, 0, 5], np.int32))
    np.testing.assert_array_equal(sub["y"], full["y"][[11, 0, 5]])
    np.testing.assert_array_equal(sub["idx"], full["idx"][[11, 0, 5]])


# --------------------------------------------------------------------------- MXFP8 activations
# The optional MXFP8 activation format (an extension: the pages quantize only the weights)
# keeps the pages' block structure, one 8-bit power-of-two scale per 32 values, with OCP FP8
# E4M3 elements.  Pinned against the format's bit fields, torch's float8_e4m3fn cast
# (round to nearest even) and a dense layer written out here.

def _torch_e4m3(a: np.ndarray) -> np.ndarray:
    """|a| < 464 rounded to E4M3 by torch's cast (values >= 464 would not saturate there)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_grid_matches_bit_fields_and_torch():
    import torch
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    fields = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        fields.append(m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    np.testing.assert_array_equal(vals, np.array(fields))
    lib_vals = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(vals, lib_vals)
    assert vals[-1] == 448.0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6
    assert math.isnan(oracle.e4m3_value(0x7F))
    assert np.all(np.diff(vals) > 0)


def test_e4m3_nearest_ties_to_even_and_saturates():
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = (vals[:-1] + vals[1:]) / 2            # exact in float64
    for i, mid in enumerate(mids):               # between codes i and i+1: the even one wins
        assert oracle.e4m3_nearest_code(mid) == (i if i % 2 == 0 else i + 1), (i, mid)
        assert oracle.e4m3_nearest_code(np.nextafter(mid, 0)) == i
        assert oracle.e4m3_nearest_code(np.nextafter(mid, 1e9)) == i + 1
    for a in (448.0, 460.0, 464.0, 1e6, float("inf")):
        assert oracle.e4m3_nearest_code(a) == 0x7E
    assert oracle.e4m3_nearest_code(0.0) == 0 and oracle.e4m3_nearest_code(2.0 ** -10) == 0
    rng = np.random.default_rng(5)
    a = np.concatenate([np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 4000)), mids[mids < 440]])
    a = a.astype(np.float32).astype(np.float64)  # values torch's float32 cast keeps exactly
    codes = np.array([oracle.e4m3_nearest_code(v) for v in a])
    np.testing.assert_array_equal(vals[codes], _torch_e4m3(a))


def test_mxfp8_block_scale_exponent():
    blocks = []
    for amax in (1.0, 255.9, 256.0, 2.0 ** -20, 3.0e38, 2.0 ** -121):
        b = np.zeros(32)
        b[7] = -amax
        b[3] = amax / 3
        blocks.append(b)
    blocks.append(np.zeros(32))
    q, exps = oracle.mxfp8_quantize(np.stack(blocks))
    expect = [-7, 0, 1, -27, 120, -122, 0]
    np.testing.assert_array_equal(exps[:, 0], expect)
    assert np.all(q[-1] == 0.0)
    for i, amax in enumerate((1.0, 255.9, 256.0, 2.0 ** -20, 3.0e38)):
        assert 128.0 <= abs(q[i, 7]) / 2.0 ** expect[i] <= 256.0


def test_mxfp8_error_bound_and_grid_membership():
    rng = np.random.default_rng(6)
    v = rng.standard_normal((200, 64)) * np.exp(rng.uniform(-8, 8, (200, 1)))
    v[:, 5] = 0.0
    q, exps = oracle.mxfp8_quantize(v)
    s = np.repeat(exps, 32, axis=1).astype(np.float64)
    r = np.abs(v) / 2.0 ** s
    top = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    bound = np.where(r >= 2.0 ** -6, 2.0 ** (top - 4), 2.0 ** -10) * 2.0 ** s
    assert np.all(np.abs(q - v) <= bound * (1 + 1e-12))
    grid = {oracle.e4m3_value(c) for c in range(0x7F)}
    assert all(abs(x) in grid for x in (q / 2.0 ** s).ravel())
    assert np.all(np.sign(q) * np.sign(v) >= 0) and np.all(q[:, 5] == 0.0)
    # idempotent: quantized values are their own quantization
    q2, exps2 = oracle.mxfp8_quantize(q)
    np.testing.assert_array_equal(q2, q)


def _mx_ref(v: np.ndarray) -> np.ndarray:
    """MXFP8 of rows of v written out here: blocks of 32 along the last axis, scale
    2^(floor(log2 amax) - 7), elements through torch's E4M3 cast."""
    out = np.empty_like(v)
    for idx in np.ndindex(v.shape[:-1]):
        for b in range(v.shape[-1] // 32):
            blk = v[idx][32 * b: 32 * b + 32]
            amax = np.abs(blk).max()
            s = (np.frexp(amax)[1] - 1 - 7) if amax > 0 else 0
            s = min(126, max(-122, s))
            out[idx][32 * b: 32 * b + 32] = _torch_e4m3(blk / 2.0 ** s) * 2.0 ** s
    return out


def test_forward_mxfp8_single_expert_is_dense_layer_on_quantized_activations():
    """E = 1, k = 1 with MXFP8 activations: xe and h quantized in 32-blocks along the
    reduction axis of the projection that reads them."""
    case = _small_case(7, 64, 96, 1, 1, seed=15)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    out = _oracle_y(case, want_h=True, act="mxfp8")
    xv = bf16_bits_to_f64(x)
    xn = xv / np.sqrt(np.mean(xv ** 2, axis=1, keepdims=True) + 1e-5) * gamma
    xe = _mx_ref(round_bf16(xn))
    gt, up = xe @ dec1[0][:cfg.I].T, xe @ dec1[0][cfg.I:].T
    h = _mx_ref(round_bf16(silu(np.minimum(gt, 7.0)) * np.clip(up, -7.0, 7.0)))
    np.testing.assert_array_equal(bf16_bits_to_f64(out["h"][:, 0, :]), h)
    np.testing.assert_allclose(out["y_f64"], xv + h @ dec2[0].T, rtol=0, atol=1e-12)
    base = _oracle_y(case)
    assert not np.array_equal(base["y_f64"], out["y_f64"])   # the format is in effect


def test_forward_mxfp8_stays_close_to_bf16():
    """MXFP8 activations move the layer's output by the E4M3 rounding only (~2^-5 relative
    per element): small against the output and far from it."""
    case = _small_case(16, 128, 128, 4, 2, seed=16)
    a, b = _oracle_y(case)["y_f64"], _oracle_y(case, act="mxfp8")["y_f64"]
    x = bf16_bits_to_f64(case[1])
    delta = np.linalg.norm(b - a) / np.linalg.norm(a - x)
    assert 1e-3 < delta < 0.1, delta


# --------------------------------------------------------------------------- MXFP4 activations
# The optional MXFP4 activation format (an extension, like MXFP8) quantizes the expert inputs
# and the SwiGLU outputs with the weights' own format and rule (ewbang.com article, 量化:
# 4-bit values, one 8-bit scale per 32).  Pinned against the already pinned weight quantizer
# and against the E2M1 bit fields written out here.

_E2M1_GRID = np.array([e2m1_from_bits(c) for c in range(8)])   # magnitudes, codes 0..7


def _mx4_ref(v: np.ndarray) -> np.ndarray:
    """MXFP4 of rows of v written out here: scale 2^(floor(log2 amax) - 2) per 32-block,
    each |v| / scale to the nearest E2M1 magnitude (the even code on a tie, 6 above 6)."""
    out = np.empty_like(v)
    for idx in np.ndindex(v.shape[:-1]):
        for b in range(v.shape[-1] // 32):
            blk = v[idx][32 * b: 32 * b + 32]
            amax = np.abs(blk).max()
            s = min(127, max(-127, np.frexp(amax)[1] - 1 - 2)) if amax > 0 else 0
            r = np.abs(blk) / 2.0 ** s
            err = np.abs(r[:, None] - _E2M1_GRID[None, :])
            best = err.min(axis=1, keepdims=True)
            cand = np.where(err == best, np.arange(8)[None, :], 99)
            even = np.where(cand % 2 == 0, cand, 99).min(axis=1)
            code = np.where(even < 99, even, cand.min(axis=1))
            code = np.where(r >= 6.0, 7, code)
            out[idx][32 * b: 32 * b + 32] = np.where(code == 0, 0.0, np.sign(blk) * _E2M1_GRID[code] * 2.0 ** s)
    return out


def test_mxfp4_activations_match_the_weight_quantizer_and_bit_fields():
    rng = np.random.default_rng(21)
    v = rng.standard_normal((64, 96)) * np.exp(rng.uniform(-6, 6, (64, 1)))
    v[0, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4) * np.where(np.arange(32) % 3, 1, -1)
    v[1, :32] = 0.0
    v = v.astype(np.float32).astype(np.float64)            # float32 values: the weight quantizer's input type
    q = oracle.mxfp4_quantize_values(v)
    np.testing.assert_array_equal(q, _mx4_ref(v))
    codes, scales = oracle.quantize(v.astype(np.float32))
    np.testing.assert_array_equal(q, oracle.dequantize(codes, scales))
    assert np.all(q[1, :32] == 0.0)
    np.testing.assert_array_equal(oracle.mxfp4_quantize_values(q), q)   # idempotent


def test_forward_mxfp4_single_expert_is_dense_layer_on_quantized_activations():
    case = _small_case(7, 64, 96, 1, 1, seed=17)
    cfg, x, gamma, rw, rb, W, dec1, dec2 = case
    out = _oracle_y(case, want_h=True, act="mxfp4")
    xv = bf16_bits_to_f64(x)
    xn = xv / np.sqrt(np.mean(xv ** 2, axis=1, keepdims=True) + 1e-5) * gamma
    xe = _mx4_ref(round_bf16(xn))
    gt, up = xe @ dec1[0][:cfg.I].T, xe @ dec1[0][cfg.I:].T
    h = _mx4_ref(round_bf16(silu(np.minimum(gt, 7.0)) * np.clip(up, -7.0, 7.0)))
    np.testing.assert_array_equal(bf16_bits_to_f64(out["h"][:, 0, :]), h)
    np.testing.assert_allclose(out["y_f64"], xv + h @ dec2[0].T, rtol=0, atol=1e-12)


def test_forward_mxfp4_moves_the_layer_more_than_mxfp8():
    case = _small_case(16, 128, 128, 4, 2, seed=18)
    a = _oracle_y(case)["y_f64"]
    x = bf16_bits_to_f64(case[1])
    d8 = np.linalg.norm(_oracle_y(case, act="mxfp8")["y_f64"] - a) / np.linalg.norm(a - x)
    d4 = np.linalg.norm(_oracle_y(case, act="mxfp4")["y_f64"] - a) / np.linalg.norm(a - x)
    assert d8 < d4 < 0.5, (d8, d4)
