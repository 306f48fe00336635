"""Out-of-range stores, checked without a sanitizer.

1. Guard bands: the workspace, y and the optional outputs live inside larger buffers filled
   with a canary byte; after each forward on the small and ragged shapes (both paths, every
   activation format, the partial and the next-norm outputs) the bands must be intact.
2. The bounds-checking build (libmoe_mxfp4_bounds.so, -DMOE_DEBUG_BOUNDS): every store at a
   computed offset (packed activation blocks, expert outputs, y, quantized weights) is
   checked against its buffer; the small shapes must run on it with a clean status word
   (no MOE_ERR_BOUNDS) and match the oracle.
"""
import numpy as np
import pytest
import torch

import mxfp4_expert_gemm_b200 as moe
import synth
from mxfp4_expert_gemm_b200 import build as libbuild
from _gpu_case import assert_parity, bf16_host, case, oracle_rows, parity_stats
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

BAND = 4096      # bytes of canary before and after each buffer (keeps 256-byte alignment)
CANARY = 0xA5
SHAPES = ["tiny", "odd", "k_eq_E", "single", "mid_ragged", "tiled_route", "wide_E", "decode_20b"]


class Banded:
    """A buffer of `nbytes` with canary bands on both sides."""

    def __init__(self, nbytes: int):
        self.n = nbytes
        self.buf = torch.full((nbytes + 2 * BAND,), CANARY, dtype=torch.uint8, device="cuda")
        self.inner = self.buf[BAND:BAND + nbytes]

    def view(self, dtype, shape):
        return self.inner.view(dtype).view(*shape)

    def intact(self) -> bool:
        b = self.buf.cpu().numpy()
        return bool(np.all(b[:BAND] == CANARY) and np.all(b[BAND + self.n:] == CANARY))


def _banded_ws(dims, T):
    w = Banded(moe.moe_workspace_bytes(dims, T))
    w.inner.zero_()   # the status word starts clear
    return w


@pytest.mark.parametrize("act", ["bf16", "mxfp8", "mxfp4"])
@pytest.mark.parametrize("path", ["gemv", "gemm"])
@pytest.mark.parametrize("name", SHAPES)
def test_guard_bands_stay_intact(name, path, act):
    c = case(SMALL[name])
    cfg = c["cfg"]
    dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path, act=act)
    args = (c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *c["W"]["gpu"])
    ws = _banded_ws(dims, cfg.T)
    y = Banded(cfg.T * cfg.d * 2)
    moe.moe_forward(dims, *args, ws.inner, y=y.view(torch.bfloat16, (cfg.T, cfg.d)))
    assert moe.moe_device_status(ws.inner) == moe.MOE_OK
    assert ws.intact() and y.intact(), "a store left its buffer"
    if act == "bf16":
        # the slice-of-I output and the next-norm outputs
        part = Banded(cfg.T * cfg.d * 4)
        moe.moe_forward_partial(dims, *args, ws.inner, y_partial=part.view(torch.float32, (cfg.T, cfg.d)))
        y2, yn = Banded(cfg.T * cfg.d * 2), Banded(cfg.T * cfg.d * 2)
        g2 = torch.ones(cfg.d, dtype=torch.float32, device="cuda")
        moe.moe_forward_norm(dims, *args, ws.inner, g2, 1e-5, y=y2.view(torch.bfloat16, (cfg.T, cfg.d)),
                             y_norm=yn.view(torch.bfloat16, (cfg.T, cfg.d)))
        assert moe.moe_device_status(ws.inner) == moe.MOE_OK
        assert ws.intact() and part.intact() and y2.intact() and yn.intact()


@pytest.fixture(scope="module")
def bounds_lib():
    path = libbuild.LIB_BOUNDS
    if not libbuild.up_to_date(path):
        libbuild.build(bounds=True)
    return path


@pytest.mark.parametrize("act", ["bf16", "mxfp4"])
@pytest.mark.parametrize("path", ["gemv", "gemm"])
@pytest.mark.parametrize("name", ["tiny", "odd", "mid_ragged", "tiled_route", "decode_20b"])
def test_bounds_checking_build_runs_clean(bounds_lib, name, path, act):
    c = case(SMALL[name])
    cfg = c["cfg"]
    ref = oracle_rows(c, act=act)
    with moe.use_library(bounds_lib):
        dims = moe.make_dims(cfg.d, cfg.I, cfg.E, cfg.k, cfg.rms_eps, cfg.swiglu_limit, path=path, act=act)
        ws = moe.new_workspace(dims, cfg.T)
        # quantize through the checked build too (its code / scale stores are checked)
        E, d, I = cfg.E, cfg.d, cfg.I
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        w = [torch.empty(sh, dtype=torch.uint8, device="cuda")
             for sh in (*moe.mxfp4_shapes(E, 2 * I, d), *moe.mxfp4_shapes(E, d, I))]
        for e in range(E):
            moe.moe_mxfp4_quantize(torch.from_numpy(synth.w1_expert(cfg, e)).cuda(), w[0][e:e + 1], w[1][e:e + 1],
                                   role="gate_up", status_word=status)
            moe.moe_mxfp4_quantize(torch.from_numpy(synth.w2_expert(cfg, e)).cuda(), w[2][e:e + 1], w[3][e:e + 1],
                                   role="down", status_word=status)
        y = moe.moe_forward(dims, c["x_dev"], c["gamma_dev"], c["rw_dev"], c["rb_dev"], *w, ws)
        assert moe.moe_device_status(ws) == moe.MOE_OK
        torch.cuda.synchronize()
        assert int(status.item()) == moe.MOE_OK
    for got, want in zip(w, c["W"]["gpu"]):
        assert torch.equal(got, want)   # the checked build quantizes bit for bit like the normal one
    assert_parity(parity_stats(bf16_host(y), ref["y"], c["x"]), f"{name}/{path}/{act} (bounds build)", act)
