"""The C-ABI library on the CPU: it loads, exports every declared symbol, and its host-side
argument checks answer before any device work (no GPU needed)."""
import ctypes

import pytest

import mxfp4_expert_gemm_b200 as moe
from mxfp4_expert_gemm_b200 import build


@pytest.fixture(scope="module")
def L():
    build.build()
    return moe.lib()


def test_every_header_symbol_is_exported(L):
    names = moe.header_functions()
    assert {"moe_mxfp4_quantize", "moe_route", "moe_forward", "moe_workspace_bytes", "moe_device_status",
            "moe_status_string", "moe_mxfp4_codes_bytes", "moe_mxfp4_scales_bytes"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_storage_sizes(L):
    # K a multiple of 128 and N of 128: exactly 4.25 bits per parameter
    assert moe.moe_mxfp4_codes_bytes(1, 256, 4096) == 256 * 4096 // 2
    assert moe.moe_mxfp4_scales_bytes(1, 256, 4096) == 256 * 4096 // 32
    # gpt-oss W1 [2I=5760][d=2880]: rows padded to 2944 codes, scale groups of 128 rows x 128
    assert moe.moe_mxfp4_codes_bytes(1, 5760, 2880) == 45 * 23 * 8192
    assert moe.moe_mxfp4_scales_bytes(1, 5760, 2880) == 45 * 23 * 512
    # W2 [d=2880][I=2880]: 22.5 row tiles -> 23
    assert moe.moe_mxfp4_codes_bytes(1, 2880, 2880) == 23 * 23 * 8192
    assert moe.moe_mxfp4_scales_bytes(1, 2880, 2880) == 23 * 23 * 512
    assert moe.moe_mxfp4_codes_bytes(32, 5760, 2880) == 32 * 45 * 23 * 8192
    assert moe.moe_mxfp4_codes_bytes(0, 5760, 2880) == 0
    assert moe.mxfp4_shapes(2, 2880, 2880) == ((2, 23, 23, 128, 64), (2, 23, 23, 512))


def test_status_strings(L):
    for s in (0, 1, 2, 3, 4, 5, 6, 7, 8):
        assert moe.status_string(s) and moe.status_string(s) != "unknown status"
    assert moe.status_string(99) == "unknown status"


def test_workspace_size_and_layout(L):
    dims = moe.make_dims(2880, 2880, 32, 4)
    n = moe.moe_workspace_bytes(dims, 4096)
    lay = moe.moe_workspace_layout(dims, 4096)
    assert lay["total"] == n and lay["status"] == 0
    offs = [lay[f] for f in moe.WS_FIELDS]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    P = 4096 * 4
    assert lay["ys"] + 4 * P * 2880 <= n
    assert moe.moe_workspace_bytes(moe.make_dims(2880, 2880, 32, 4, block=16), 16) == 0
    # MXFP8 activations: one E4M3 row per token, tiles of twice the tokens, same block size
    mx = moe.moe_workspace_layout(moe.make_dims(2880, 2880, 32, 4, act="mxfp8"), 4096)
    assert mx["status"] == 0 and mx["total"] <= n
    assert moe.moe_workspace_bytes(moe.make_dims(2880, 2880, 32, 4, act=9), 16) == 0


def _call_forward(L, dims, T, ptr=256, ws_bytes=1 << 40):
    p = ctypes.c_void_p(ptr)
    return L.moe_forward(ctypes.byref(dims), T, p, p, p, p, p, p, p, p, ctypes.c_void_p(ptr + 4096), None, None,
                         None, p, ws_bytes, None)


def test_argument_checks_before_device(L):
    ok = moe.make_dims(2880, 2880, 32, 4)
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, block=16), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # d and I in whole multiples of 64 (the library's rule; the pages' block is 32): odd
    # multiples of 32 are refused, for either dimension, before anything runs
    assert _call_forward(L, moe.make_dims(2880 + 32, 2880, 32, 4), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880 + 32, 32, 4), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(96, 160, 4, 2), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert moe.moe_workspace_bytes(moe.make_dims(96, 128, 4, 2), 4) == 0
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 33), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 300, 4), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 4, 5), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, path=9), 4) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, rms_eps=-1.0), 4) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, act=7), 4) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, ok, -1) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, ok, 4, ptr=8) == moe.MOE_ERR_INVALID_ARG          # misaligned
    assert _call_forward(L, ok, 4, ptr=0) == moe.MOE_ERR_INVALID_ARG          # null
    assert _call_forward(L, ok, 4096, ws_bytes=1024) == moe.MOE_ERR_WORKSPACE
    assert L.moe_forward(None, 4, *([None] * 13), 0, None) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, ok, 4, ptr=16) == moe.MOE_ERR_INVALID_ARG         # codes need 32-byte alignment
    p = ctypes.c_void_p(256)
    assert L.moe_mxfp4_quantize(p, 1, 64, 48, 0, p, p, None, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_mxfp4_quantize(None, 1, 64, 64, 0, p, p, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_mxfp4_quantize(p, 1, 64, 64, 7, p, p, None, None) == moe.MOE_ERR_INVALID_ARG     # bad role
    assert L.moe_mxfp4_quantize(p, 1, 64, 64, 1, p, p, None, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE  # I = 32
    assert L.moe_mxfp4_quantize(p, 1, 128, 64, 1, ctypes.c_void_p(272), p, None, None) == moe.MOE_ERR_INVALID_ARG


def test_no_device_is_an_error_not_a_fallback(L):
    """With valid arguments and no usable GPU the call fails; there is no CPU path."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _call_forward(L, moe.make_dims(128, 128, 4, 2), 4)
    assert st in (moe.MOE_ERR_CUDA, moe.MOE_ERR_DEVICE)


def test_no_alloc_argument_checks_match_moe_forward(L):
    """moe_forward_no_alloc answers argument errors with moe_forward's codes, before any
    device work."""
    p = ctypes.c_void_p(256)

    def call(dims, T):
        return L.moe_forward_no_alloc(ctypes.byref(dims) if dims is not None else None, T, p, p, p, p, p, p, p, p,
                                      ctypes.c_void_p(256 + 4096), None, None)

    for dims, T in ((moe.make_dims(2880, 2880, 32, 4, path=9), 4), (moe.make_dims(2880, 2880, 32, 4, act=3), 4),
                    (moe.make_dims(2880, 2880, 32, 4), -1), (moe.make_dims(2880, 2880, 32, 4, block=16), 4),
                    (moe.make_dims(2880 + 32, 2880, 32, 4), 4), (moe.make_dims(2880, 2880, 4, 5), 4)):
        assert call(dims, T) == _call_forward(L, dims, T), (dims.path, dims.act_format, T)
    assert call(None, 4) == moe.MOE_ERR_INVALID_ARG
    assert call(moe.make_dims(2880, 2880, 32, 4), 4096) == moe.MOE_ERR_WORKSPACE   # beyond the 16 MiB scratch


def _call_host(L, dims, T, ptr=256, ws_bytes=1 << 40, chunk=0, x_dev=None, y_dev=None, hp=4096):
    p = ctypes.c_void_p(ptr)
    xd = ctypes.c_void_p(ptr if x_dev is None else x_dev)
    yd = ctypes.c_void_p(ptr + 8192 if y_dev is None else y_dev)
    h = ctypes.c_void_p(hp)
    return L.moe_forward_host(ctypes.byref(dims) if dims is not None else None, T, h, h, xd, yd, p, p, None,
                              p, p, p, p, p, ws_bytes, chunk, None, None, None)


def test_host_entry_argument_checks_before_device(L):
    """moe_forward_host refuses bad arguments before it enqueues anything (no GPU needed)."""
    ok = moe.make_dims(2880, 2880, 32, 4)
    assert _call_host(L, None, 4) == moe.MOE_ERR_INVALID_ARG
    assert _call_host(L, ok, -1) == moe.MOE_ERR_INVALID_ARG
    assert _call_host(L, ok, 0) == moe.MOE_OK                                    # nothing to do
    assert _call_host(L, ok, 16, chunk=-1) == moe.MOE_ERR_INVALID_ARG
    assert _call_host(L, ok, 16, hp=0) == moe.MOE_ERR_INVALID_ARG                # null host buffers
    assert _call_host(L, ok, 16, x_dev=512, y_dev=512) == moe.MOE_ERR_INVALID_ARG  # x_dev aliases y_dev
    assert _call_host(L, ok, 16, x_dev=520) == moe.MOE_ERR_INVALID_ARG          # misaligned x_dev
    assert _call_host(L, ok, 16, ptr=16) == moe.MOE_ERR_INVALID_ARG             # codes need 32-byte alignment
    assert _call_host(L, moe.make_dims(2880 + 32, 2880, 32, 4), 16) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # the workspace must hold a chunk: the whole batch's is more than enough, a chunk's
    # exactly enough, a byte less is refused
    T, c = 8192, moe.moe_host_chunk_tokens(ok, 8192)
    need = max(moe.moe_workspace_bytes(ok, c), moe.moe_workspace_bytes(ok, T - (T + c - 1) // c * c + c))
    assert _call_host(L, ok, T, ws_bytes=need - 1) == moe.MOE_ERR_WORKSPACE
    assert _call_host(L, ok, T, ws_bytes=moe.moe_workspace_bytes(ok, 100), chunk=100) != moe.MOE_ERR_WORKSPACE
    assert _call_host(L, ok, T, ws_bytes=moe.moe_workspace_bytes(ok, 99), chunk=100) == moe.MOE_ERR_WORKSPACE


def test_host_entry_chunk_choice(L):
    """One chunk on the small-batch path and below 4096 tokens; else two to four chunks of at
    least 2048 tokens that cover the batch."""
    d20, d120 = moe.make_dims(2880, 2880, 32, 4), moe.make_dims(2880, 2880, 128, 4)
    assert moe.moe_host_chunk_tokens(d20, 16) == 16
    assert moe.moe_host_chunk_tokens(d20, 4095) == 4095
    assert moe.moe_host_chunk_tokens(d20, 4096) == 2048
    assert moe.moe_host_chunk_tokens(d120, 16384) == 4096
    assert moe.moe_host_chunk_tokens(d120, 8192) == 2048
    assert moe.moe_host_chunk_tokens(d120, 6000) == 3000
    # few tokens per expert (E = 256, top-1: 16 per expert at 4096 tokens): one chunk
    assert moe.moe_host_chunk_tokens(moe.make_dims(2880, 2880, 256, 1), 4096) == 4096
    for T in (4096, 5000, 9999, 16384, 100000):
        c = moe.moe_host_chunk_tokens(d120, T)
        n = (T + c - 1) // c
        assert 2 <= n <= 4 and c >= 2048 and (n - 1) * c < T
    assert L.moe_host_chunk_tokens(None, 16) == -1


def test_no_device_host_entry_is_an_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _call_host(L, moe.make_dims(128, 128, 4, 2), 4) in (moe.MOE_ERR_CUDA, moe.MOE_ERR_DEVICE)
