"""Tensor parallelism over the intermediate features, on the CPU (oracle, gloo ranks).

A rank holds, for every expert, the gate rows [i0, i1) and up rows [I + i0, I + i1) of W1
and the columns [i0, i1) of W2 (slices of whole 64-feature blocks), runs the layer on that
slice without the residual, and the ranks all-reduce their partial outputs.  The sum plus
x must be the whole layer: the expert MLP is separable over its intermediate features
(each feature of h depends on its own gate and up rows; the down projection sums over the
features), and slicing the fp32 weights before quantizing gives the same MXFP4 blocks as
slicing the quantized matrices, because the slices start on 32-value block boundaries.
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CFG = dict(name="tp_small", T=12, d=128, I=384, E=4, k=2, seed=3)


def _slice_weights(cfg, i0, i1):
    """Oracle-layout MXFP4 weights of one slice of the intermediate features, all experts."""
    import oracle
    import synth
    E, d, I = cfg.E, cfg.d, cfg.I
    Ir = i1 - i0
    out = (np.empty((E, 2 * Ir, d // 2), np.uint8), np.empty((E, 2 * Ir, d // 32), np.uint8),
           np.empty((E, d, Ir // 2), np.uint8), np.empty((E, d, Ir // 32), np.uint8))
    for e in range(E):
        w1 = synth.w1_expert(cfg, e)
        w1s = np.concatenate([w1[i0:i1], w1[I + i0:I + i1]])
        w2s = np.ascontiguousarray(synth.w2_expert(cfg, e)[:, i0:i1])
        out[0][e], out[1][e] = oracle.quantize(w1s)
        out[2][e], out[3][e] = oracle.quantize(w2s)
    return out


def _partial(cfg, x, i0, i1):
    """The slice's share of the expert mix (no residual), fp64."""
    import oracle
    import synth
    W = _slice_weights(cfg, i0, i1)
    r = oracle.moe_forward(x, synth.norm_weight(cfg), synth.router_weight(cfg), synth.router_bias(cfg), *W,
                           I=i1 - i0, k=cfg.k)
    return r["y_f64"] - synth.bf16_to_f32(x).astype(np.float64), r["idx"]


def _full(cfg, x):
    import oracle
    import synth
    from _inputs import oracle_weights
    return oracle.moe_forward(x, synth.norm_weight(cfg), synth.router_weight(cfg), synth.router_bias(cfg),
                              *oracle_weights(cfg), I=cfg.I, k=cfg.k)


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import synth
    from mxfp4_expert_gemm_b200 import intermediate_slices
    cfg = synth.MoEConfig(**CFG)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    x = synth.hidden(cfg)   # every rank holds the whole batch
    i0, i1 = intermediate_slices(cfg.I, world)[rank]
    part, idx = _partial(cfg, x, i0, i1)
    t = torch.from_numpy(part)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    idx_all = [None] * world
    dist.all_gather_object(idx_all, idx.tolist())
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t.numpy(), idx_all, (i0, i1)))


def test_two_gloo_ranks_sum_their_slices_to_the_whole_layer():
    sys.path.insert(0, ROOT)
    import synth
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=300) for _ in range(world)], key=lambda o: o[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = synth.MoEConfig(**CFG)
    x = synth.hidden(cfg)
    full = _full(cfg, x)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    assert [o[3] for o in out] == [(0, 192), (192, 384)]
    for rank, s, idx_all, _ in out:
        # every rank routed the same tokens to the same experts
        assert idx_all[0] == idx_all[1] == full["idx"].tolist()
        y = xf + s
        scale = np.abs(full["y_f64"] - xf).max()
        assert np.abs(y - full["y_f64"]).max() <= 1e-12 * scale, rank


@pytest.mark.parametrize("G", [1, 3, 6])
def test_slices_of_whole_blocks_cover_I_and_sum_to_the_layer(G):
    sys.path.insert(0, ROOT)
    import synth
    from mxfp4_expert_gemm_b200 import intermediate_slices
    cfg = synth.MoEConfig(**CFG)
    sl = intermediate_slices(cfg.I, G)
    assert sl[0][0] == 0 and sl[-1][1] == cfg.I
    assert all(a1 == b0 for (_, a1), (b0, _) in zip(sl, sl[1:]))
    assert all((i1 - i0) % 64 == 0 and i1 > i0 for i0, i1 in sl)
    x = synth.hidden(cfg)
    total = sum(_partial(cfg, x, i0, i1)[0] for i0, i1 in sl)
    full = _full(cfg, x)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    assert np.abs(xf + total - full["y_f64"]).max() <= 1e-12 * np.abs(full["y_f64"] - xf).max()


def test_slicing_rejects_widths_that_are_not_whole_blocks():
    sys.path.insert(0, ROOT)
    from mxfp4_expert_gemm_b200 import intermediate_slices
    assert intermediate_slices(2880, 2) == [(0, 1472), (1472, 2880)]
    with pytest.raises(ValueError):
        intermediate_slices(2880, 46)
    with pytest.raises(ValueError):
        intermediate_slices(2880 + 32, 2)
