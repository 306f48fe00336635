"""GPU parity of the slice-of-I forward (tensor parallelism over the intermediate features)
and of the forward that also writes the next block's RMSNorm of its output.

Slices: every slice's weights are quantized by the library from the sliced fp32 weights;
each slice's partial output is compared with the oracle's share of the expert mix for that
slice, and the slices' sum (added on the device, standing in for the all-reduce of several
GPUs) is finished by moe_residual_norm and compared with the oracle's whole layer.

Next-block RMSNorm: y must equal moe_forward's y bit for bit (the same sums in the same
order), and y_norm is compared with the oracle's RMSNorm of the oracle's own output.
"""
import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import oracle
import synth
from _gpu_case import assert_parity, bf16_dev, bf16_host, case, oracle_rows, parity_stats
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


def _slice_case(cfg, i0, i1):
    """Library (GPU) and oracle MXFP4 weights of one slice [i0, i1) of the features."""
    E, d, I = cfg.E, cfg.d, cfg.I
    Ir = i1 - i0
    s1c, s1s = moe.mxfp4_shapes(E, 2 * Ir, d)
    s2c, s2s = moe.mxfp4_shapes(E, d, Ir)
    g = [torch.empty(sh, dtype=torch.uint8, device="cuda") for sh in (s1c, s1s, s2c, s2s)]
    o = (np.empty((E, 2 * Ir, d // 2), np.uint8), np.empty((E, 2 * Ir, d // 32), np.uint8),
         np.empty((E, d, Ir // 2), np.uint8), np.empty((E, d, Ir // 32), np.uint8))
    for e in range(E):
        w1 = synth.w1_expert(cfg, e)
        w1s = np.ascontiguousarray(np.concatenate([w1[i0:i1], w1[I + i0:I + i1]]))
        w2s = np.ascontiguousarray(synth.w2_expert(cfg, e)[:, i0:i1])
        moe.moe_mxfp4_quantize(torch.from_numpy(w1s).cuda(), g[0][e:e + 1], g[1][e:e + 1], role="gate_up")
        moe.moe_mxfp4_quantize(torch.from_numpy(w2s).cuda(), g[2][e:e + 1], g[3][e:e + 1], role="down")
        o[0][e], o[1][e] = oracle.quantize(w1s)
        o[2][e], o[3][e] = oracle.quantize(w2s)
    return g, o


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("name,path,G", [("decode_20b", "auto", 2), ("mid_ragged", "gemm", 2),
                                         ("mid_ragged", "gemv", 3), ("odd", "gemm", 5)])
def test_slices_of_I_sum_to_the_layer(name, path, G):
    c = case(SMALL[name])
    cfg = c["cfg"]
    x = c["x"]
    xf = synth.bf16_to_f32(x).astype(np.float64)
    total = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    for i0, i1 in moe.intermediate_slices(cfg.I, G):
        g, o = _slice_case(cfg, i0, i1)
        dims = moe.make_dims(cfg.d, i1 - i0, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path)
        ws = moe.new_workspace(dims, cfg.T)
        part = moe.moe_forward_partial(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *g, ws)
        assert moe.moe_device_status(ws) == moe.MOE_OK
        ref = oracle.moe_forward(x, c["gamma"], c["rw"], c["rb"], *o, I=i1 - i0, k=cfg.k, eps=cfg.rms_eps,
                                 limit=cfg.swiglu_limit)
        want = ref["y_f64"] - xf
        got = part.cpu().numpy().astype(np.float64)
        assert _rel(got, want) <= 1e-2, (i0, i1, _rel(got, want))
        total += part   # the all-reduce of the ranks' partial outputs
    y = moe.moe_residual_norm(c["x_dev"], total)
    ref_full = oracle_rows(c)
    st = parity_stats(bf16_host(y), ref_full["y"], x)
    assert_parity(st, f"{name}/{path}/G={G}")
    assert st["delta_rel_fro"] <= 2.5e-2, st


@pytest.mark.parametrize("path", ["gemv", "gemm"])
@pytest.mark.parametrize("name", ["tiny", "decode_20b", "odd", "mid_ragged", "tiled_route"])
def test_forward_with_next_block_norm(name, path):
    c = case(SMALL[name])
    cfg = c["cfg"]
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path)
    gamma2 = synth.normal_f32(cfg.seed + 101, 2, 0, cfg.d, 1.0, 0.1)   # the next block's RMSNorm weight
    g2 = torch.from_numpy(gamma2).cuda()
    args = (c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    ws = moe.new_workspace(dims, cfg.T)
    y, y_norm = moe.moe_forward_norm(dims, *args, ws, g2, 1e-5)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    y_plain = moe.moe_forward(dims, *args, ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    np.testing.assert_array_equal(bf16_host(y), bf16_host(y_plain))
    ref = oracle_rows(c)
    assert_parity(parity_stats(bf16_host(y), ref["y"], c["x"]), f"{name}/{path}")
    want = oracle.next_block_norm(ref["y"], gamma2, 1e-5)
    got = bf16_host(y_norm)
    gf, wf = synth.bf16_to_f32(got).astype(np.float64), synth.bf16_to_f32(want).astype(np.float64)
    assert _rel(gf, wf) <= 1e-2
    assert np.abs(gf - wf).max() <= 5e-2 * np.sqrt(np.mean(wf * wf))


def test_residual_norm_alone():
    rng = np.random.default_rng(9)
    T, d = 37, 2880
    x = oracle.to_bf16(rng.standard_normal((T, d)))
    s = (rng.standard_normal((T, d)) * 0.3).astype(np.float32)
    gamma = (1 + 0.1 * rng.standard_normal(d)).astype(np.float32)
    y, y_norm = moe.moe_residual_norm(bf16_dev(x), torch.from_numpy(s).cuda(), torch.from_numpy(gamma).cuda(), 1e-5)
    want_y = oracle.to_bf16(synth.bf16_to_f32(x).astype(np.float64) + s.astype(np.float64))
    got_y = bf16_host(y)
    # fp32 add then one rounding vs the exact sum rounded once: at most one bf16 step apart
    gy, wy = synth.bf16_to_f32(got_y).astype(np.float64), synth.bf16_to_f32(want_y).astype(np.float64)
    assert np.all(np.abs(gy - wy) <= np.abs(wy) * 2.0 ** -7)
    assert np.mean(got_y == want_y) >= 0.999
    wn = synth.bf16_to_f32(oracle.next_block_norm(want_y, gamma, 1e-5)).astype(np.float64)
    gn = synth.bf16_to_f32(bf16_host(y_norm)).astype(np.float64)
    assert _rel(gn, wn) <= 1e-3
    # y alone, no norm
    y_only = moe.moe_residual_norm(bf16_dev(x), torch.from_numpy(s).cuda())
    np.testing.assert_array_equal(bf16_host(y_only), got_y)


@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_combine_adds_only_the_splits_of_this_call(path):
    """The down GEMM chooses its reduction-axis splits per call; the combine and the
    next-norm pass must add exactly those partial-sum planes.  Planes past them (left by an
    earlier call that split further, or never written) hold garbage here and must not
    enter y."""
    c = case(SMALL["decode_20b"])
    cfg = c["cfg"]
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path)
    ws = moe.new_workspace(dims, cfg.T)
    lay = moe.moe_workspace_layout(dims, cfg.T)
    args = (c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    ws[lay["ys"]:lay["total"]].fill_(0x4B)   # every plane: about 1.3e7 per value
    y = moe.moe_forward(dims, *args, ws)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    assert_parity(parity_stats(bf16_host(y), oracle_rows(c)["y"], c["x"]), f"garbage planes/{path}")
    ws[lay["ys"]:lay["total"]].fill_(0x4B)
    g2 = torch.ones(cfg.d, dtype=torch.float32, device="cuda")
    y2, _ = moe.moe_forward_norm(dims, *args, ws, g2, 1e-5)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    np.testing.assert_array_equal(bf16_host(y2), bf16_host(y))
