"""GPU parity at the full workload sizes: every output row against the CPU oracle.

The three full-size workloads (gpt-oss-20b prefill, T = 4096, E = 32; gpt-oss-120b,
T = 8192, E = 128; the Zipf-skewed 120b batch, T = 16384) run through the C ABI and
are compared with the oracle on every token, on the exact (bf16-activation) layer.
The routing and the grouping (counts, offsets, the (expert, token)-sorted pair list,
the token tiles of both paths) are compared bit for bit.  The MXFP8 activation format
and the MXFP4 activation formats are checked on a deterministic token set that holds the
first and the last token of every token tile of every expert.

The oracle is computed once per workload (all host cores, about a minute for the
20b prefill batch and a few minutes for the skewed batch) and shared by the paths.
"""
import functools

import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import oracle
import synth
from _gpu_case import assert_parity, bf16_host, case, oracle_rows, parity_stats, run_gpu, tile_tokens

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

C = synth.CONFIGS
FULL = ["prefill_20b", "moe_120b", "skew_120b"]


@functools.lru_cache(maxsize=1)
def oracle_all_rows(name: str):
    """The oracle's layer output on every token of workload ``name`` (bf16 activations)."""
    return oracle_rows(case(C[name]))


def expected_tiles(counts: np.ndarray, bt: int):
    """Token tiles of the expert-sorted pair list: each expert's rows cut into runs of bt,
    experts in order -> (tiles [n, 3] = (expert, first row, rows), first tile of each expert)."""
    offsets = np.concatenate([[0], np.cumsum(counts)])
    tiles, base = [], []
    for e, c in enumerate(counts.tolist()):
        base.append(len(tiles))
        for i in range(0, c, bt):
            tiles.append((e, offsets[e] + i, min(bt, c - i)))
    return np.array(tiles, np.int64).reshape(-1, 3), np.array(base, np.int64)


def tile_cover_tokens(idx: np.ndarray, E: int, bt: int) -> np.ndarray:
    """Tokens holding the first and the last pair of every token tile of every expert."""
    g = oracle.group(idx, E)
    k = idx.shape[1]
    toks = set()
    for e in range(E):
        lo, hi = int(g["offsets"][e]), int(g["offsets"][e + 1])
        for r0 in range(lo, hi, bt):
            r1 = min(hi, r0 + bt) - 1
            toks.add(int(g["perm"][r0]) // k)
            toks.add(int(g["perm"][r1]) // k)
    return np.array(sorted(toks), np.int32)


@pytest.mark.parametrize("name", FULL)
def test_full_size_routing_and_grouping_bit_exact(name):
    """moe_route at full size: expert sets, counts, offsets and the pair order against
    the oracle; the workspace's token tiles of both paths against the tiles the counts
    define."""
    c = case(C[name])
    cfg = c["cfg"]
    ref = c["route"]
    gr = oracle.group(ref["idx"], cfg.E)
    for path in ("gemm", "gemv"):
        dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path)
        ws = moe.new_workspace(dims, cfg.T)
        out = moe.moe_route(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], ws)
        assert moe.moe_device_status(ws) == moe.MOE_OK
        idx = out["topk_idx"].cpu().numpy()
        np.testing.assert_array_equal(np.sort(idx, 1), np.sort(ref["idx"], 1))
        np.testing.assert_array_equal(out["counts"].cpu().numpy(), gr["counts"])
        np.testing.assert_array_equal(out["offsets"].cpu().numpy(), gr["offsets"])
        perm = out["perm"].cpu().numpy()
        # the pair order is unique as (token, expert); slots may differ only by ties
        t_g, t_o = perm // cfg.k, gr["perm"] // cfg.k
        np.testing.assert_array_equal(t_g, t_o)
        np.testing.assert_array_equal(idx[t_g, perm % cfg.k], ref["idx"][t_o, gr["perm"] % cfg.k])
        # token tiles
        bt = tile_tokens(path)
        want, want_base = expected_tiles(gr["counts"], bt)
        view = lambda f, dt, sh: moe.workspace_view(ws, dims, cfg.T, f, dt, sh).cpu().numpy()
        assert int(view("ntiles", torch.int32, (1,))[0]) == len(want)
        tiles = view("tiles", torch.int32, (len(want), 4))[:, :3]
        np.testing.assert_array_equal(tiles, want)
        np.testing.assert_array_equal(view("tile_base", torch.int32, (cfg.E,)), want_base)
        # inv is perm's inverse
        inv = view("inv", torch.int32, (cfg.pairs,))
        np.testing.assert_array_equal(inv[perm], np.arange(cfg.T * cfg.k))


@pytest.mark.parametrize("name,path", [
    ("prefill_20b", "gemm"), ("prefill_20b", "gemv"),
    ("moe_120b", "gemm"),
    ("skew_120b", "gemm"), ("skew_120b", "gemv"),
])
def test_full_size_every_row(name, path):
    """The whole layer on every token of the workload against the oracle."""
    c = case(C[name])
    cfg = c["cfg"]
    assert c["W"]["mismatches"] == 0
    g = run_gpu(c, path)
    assert g["status"] == moe.MOE_OK, moe.status_string(g["status"])
    idx = g["routing"]["topk_idx"].cpu().numpy()
    np.testing.assert_array_equal(np.sort(idx, 1), np.sort(c["route"]["idx"], 1))
    np.testing.assert_array_equal(g["routing"]["counts"].cpu().numpy(),
                                  np.bincount(c["route"]["idx"].ravel(), minlength=cfg.E))
    ref = oracle_all_rows(name)
    st = parity_stats(bf16_host(g["y"]), ref["y"], c["x"])
    assert_parity(st, f"{name}/{path}")
    assert st["delta_rel_fro"] <= 2.5e-2, st
    # the layer's tolerance token by token: a wrong tile cannot hide in the batch's norm
    yg = synth.bf16_to_f32(bf16_host(g["y"])).astype(np.float64)
    yr = synth.bf16_to_f32(ref["y"]).astype(np.float64)
    row_err = np.linalg.norm(yg - yr, axis=1) / np.linalg.norm(yr, axis=1)
    assert row_err.max() <= 1e-2, (int(row_err.argmax()), float(row_err.max()))


@pytest.mark.parametrize("name,path,act", [("prefill_20b", "gemm", "mxfp8"), ("moe_120b", "gemm", "mxfp8"),
                                           ("prefill_20b", "gemv", "mxfp8"), ("prefill_20b", "gemm", "mxfp4"),
                                           ("skew_120b", "gemm", "mxfp4"), ("prefill_20b", "gemv", "mxfp4")])
def test_full_size_low_precision_tile_cover(name, path, act):
    """MXFP8 / MXFP4 activations at full size, on the first and last token of every token tile."""
    c = case(C[name])
    cfg = c["cfg"]
    g = run_gpu(c, path, act=act)
    assert g["status"] == moe.MOE_OK, moe.status_string(g["status"])
    np.testing.assert_array_equal(np.sort(g["routing"]["topk_idx"].cpu().numpy(), 1),
                                  np.sort(c["route"]["idx"], 1))
    toks = tile_cover_tokens(c["route"]["idx"], cfg.E, tile_tokens(path, act))
    ref = oracle_rows(c, tokens=toks, act=act)
    st = parity_stats(bf16_host(g["y"])[toks], ref["y"], c["x"][toks])
    assert_parity(st, f"{name}/{path}/{act}", act)
