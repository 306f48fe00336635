"""moe_forward_host: the layer from host memory to host memory, in chunks whose copies run
on their own streams.  Every chunking gives the layer (against the oracle); one chunk is
moe_forward's launches bit for bit; a CUDA graph of the call replays it exactly."""
import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import synth
from _gpu_case import assert_parity, bf16_host, case, oracle_rows, parity_stats
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

SHAPES = {**{n: SMALL[n] for n in ("tiny", "odd", "mid_ragged", "tiled_route", "decode_20b")},
          # enough tokens for the library to cut the batch in two (GEMM path)
          "two_chunks": synth.MoEConfig("two_chunks", T=4100, d=256, I=128, E=8, k=2)}


def _dims(cfg):
    return moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit)


def _workspace(dims, T, chunk):
    c = min(chunk or moe.moe_host_chunk_tokens(dims, T), T)
    last = T - (T - 1) // c * c
    return torch.zeros(max(moe.moe_workspace_bytes(dims, c), moe.moe_workspace_bytes(dims, last)),
                       dtype=torch.uint8, device="cuda")


def _run(c, dims, chunk, streams=True):
    x_host = c["x_dev"].cpu().pin_memory()
    x_dev, y_dev = torch.empty_like(c["x_dev"]), torch.empty_like(c["x_dev"])
    ws = _workspace(dims, c["cfg"].T, chunk)
    h2d, d2h = (torch.cuda.Stream(), torch.cuda.Stream()) if streams else (None, None)
    y_host = moe.moe_forward_host(dims, x_host, c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws,
                                  x_dev, y_dev, chunk_tokens=chunk, h2d_stream=h2d, d2h_stream=d2h)
    launches = moe.last_launch_count()
    torch.cuda.current_stream().synchronize()
    assert moe.moe_device_status(ws) == moe.MOE_OK
    return y_host, launches


@pytest.mark.parametrize("chunk", [0, 1, 7, 64])
@pytest.mark.parametrize("name", list(SHAPES))
def test_host_entry_matches_oracle(name, chunk):
    c = case(SHAPES[name])
    cfg = c["cfg"]
    if chunk == 1 and cfg.T > 400:
        pytest.skip("one-token chunks of a large batch: thousands of calls")
    dims = _dims(cfg)
    y_host, launches = _run(c, dims, chunk)
    ref = oracle_rows(c)
    got = y_host.view(torch.int16).numpy().view(np.uint16)
    st = parity_stats(got, ref["y"], c["x"])
    assert_parity(st, f"{name}/chunk {chunk}")
    assert st["delta_rel_fro"] <= 2.5e-2, st
    assert launches > 0


@pytest.mark.parametrize("name", ["tiny", "mid_ragged", "decode_20b"])
def test_one_chunk_is_moe_forward(name):
    """One chunk: the same kernels on the same tokens, so y is moe_forward's bit for bit (with
    and without the copy streams, which one chunk does not use)."""
    c = case(SHAPES[name])
    cfg = c["cfg"]
    dims = _dims(cfg)
    ws = moe.new_workspace(dims, cfg.T)
    y = moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws)
    n_fwd = moe.last_launch_count()
    want = bf16_host(y)
    for streams in (True, False):
        y_host, launches = _run(c, dims, cfg.T, streams)
        np.testing.assert_array_equal(y_host.view(torch.int16).numpy().view(np.uint16), want)
        assert launches == n_fwd


def test_chunks_replay_from_a_cuda_graph():
    """The chunked call with its two copy streams captured into a graph: replays write y_host
    exactly as the eager call did."""
    c = case(SHAPES["mid_ragged"])
    cfg = c["cfg"]
    dims = _dims(cfg)
    chunk = 64   # 64 + 64 + 64 + 8 tokens
    x_host = c["x_dev"].cpu().pin_memory()
    x_dev, y_dev = torch.empty_like(c["x_dev"]), torch.empty_like(c["x_dev"])
    ws = _workspace(dims, cfg.T, chunk)
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    args = (dims, x_host, c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], ws, x_dev, y_dev)
    eager = moe.moe_forward_host(*args, chunk_tokens=chunk, h2d_stream=h2d, d2h_stream=d2h)
    torch.cuda.synchronize()
    want = eager.clone()
    y_host = torch.zeros_like(eager).pin_memory()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_forward_host(*args, y_host=y_host, chunk_tokens=chunk, h2d_stream=h2d, d2h_stream=d2h)
    torch.cuda.synchronize()
    for _ in range(2):
        y_host.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y_host.view(torch.int16), want.view(torch.int16))
    del g
    assert moe.moe_device_status(ws) == moe.MOE_OK


def test_host_entry_argument_errors():
    c = case(SHAPES["tiny"])
    cfg = c["cfg"]
    dims = _dims(cfg)
    x_host = c["x_dev"].cpu().pin_memory()
    x_dev, y_dev = torch.empty_like(c["x_dev"]), torch.empty_like(c["x_dev"])
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward_host(dims, x_host, c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], small,
                             x_dev, y_dev)
    assert e.value.status == moe.MOE_ERR_WORKSPACE
    with pytest.raises(TypeError):
        moe.moe_forward_host(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"], small,
                             x_dev, y_dev)
