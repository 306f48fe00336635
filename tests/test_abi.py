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
    assert moe.moe_mxfp4_codes_bytes(1, 5760, 2880) == 8_294_400
    assert moe.moe_mxfp4_scales_bytes(1, 5760, 2880) == 518_400
    assert moe.moe_mxfp4_codes_bytes(32, 5760, 2880) == 32 * 8_294_400
    assert moe.moe_mxfp4_codes_bytes(0, 5760, 2880) == 0


def test_status_strings(L):
    for s in range(9):
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


def _call_forward(L, dims, T, ptr=16, ws_bytes=1 << 40):
    p = ctypes.c_void_p(ptr)
    return L.moe_forward(ctypes.byref(dims), T, p, p, p, p, p, p, p, p, ctypes.c_void_p(ptr + 4096), None, None,
                         None, p, ws_bytes, None)


def test_argument_checks_before_device(L):
    ok = moe.make_dims(2880, 2880, 32, 4)
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, block=16), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880 + 32, 2880, 32, 4), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 33), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 300, 4), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 4, 5), 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, path=9), 4) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, moe.make_dims(2880, 2880, 32, 4, rms_eps=-1.0), 4) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, ok, -1) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(L, ok, 4, ptr=8) == moe.MOE_ERR_INVALID_ARG          # misaligned
    assert _call_forward(L, ok, 4, ptr=0) == moe.MOE_ERR_INVALID_ARG          # null
    assert _call_forward(L, ok, 4096, ws_bytes=1024) == moe.MOE_ERR_WORKSPACE
    assert L.moe_forward(None, 4, *([None] * 13), 0, None) == moe.MOE_ERR_INVALID_ARG
    p = ctypes.c_void_p(16)
    assert L.moe_mxfp4_quantize(p, 1, 64, 48, p, p, None, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_mxfp4_quantize(None, 1, 64, 64, p, p, None, None) == moe.MOE_ERR_INVALID_ARG


def test_no_device_is_an_error_not_a_fallback(L):
    """With valid arguments and no usable GPU the call fails; there is no CPU path."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _call_forward(L, moe.make_dims(128, 128, 4, 2), 4)
    assert st in (moe.MOE_ERR_CUDA, moe.MOE_ERR_DEVICE)
