"""Python binding of ``libmoe_mxfp4.so``: the B200 MoE layer with MXFP4 experts.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  The C ABI and
its contract are in ``include/moe_mxfp4.h``; the functions here carry the same
names.  There is no fallback: if the library is missing or the device is not
sm_100, the calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import re
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_mxfp4.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "moe_mxfp4.h")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_NONFINITE = 6
MOE_ERR_BOUNDS = 7
MOE_ERR_DEVICE = 8

MOE_PATH_AUTO = 0
MOE_PATH_GEMV = 1
MOE_PATH_GEMM = 2
PATHS = {"auto": MOE_PATH_AUTO, "gemv": MOE_PATH_GEMV, "gemm": MOE_PATH_GEMM}

MOE_ACT_BF16 = 0
MOE_ACT_MXFP8 = 1
MOE_ACT_MXFP4 = 2
ACT_FORMATS = {"bf16": MOE_ACT_BF16, "mxfp8": MOE_ACT_MXFP8, "mxfp4": MOE_ACT_MXFP4}

MOE_WEIGHT_PLAIN = 0
MOE_WEIGHT_GATE_UP = 1
ROLES = {"plain": MOE_WEIGHT_PLAIN, "down": MOE_WEIGHT_PLAIN, "gate_up": MOE_WEIGHT_GATE_UP}


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class moe_dims(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("block", ctypes.c_int32), ("rms_eps", ctypes.c_float), ("swiglu_limit", ctypes.c_float),
                ("path", ctypes.c_int32), ("act_format", ctypes.c_int32)]


def make_dims(d: int, I: int, E: int, top_k: int, rms_eps: float = 1e-5, swiglu_limit: float = 7.0,
              path: int | str = MOE_PATH_AUTO, block: int = 32, act: int | str = MOE_ACT_BF16) -> moe_dims:
    if isinstance(path, str):
        path = PATHS[path]
    if isinstance(act, str):
        act = ACT_FORMATS[act]
    return moe_dims(d, I, E, top_k, block, rms_eps, swiglu_limit, path, act)


_lib = None
_lock = threading.Lock()


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mxfp4_expert_gemm_b200.build`")
            _lib = load_library(LIB_PATH)
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Run the calls inside the block on another build of the library (for example the
    bounds-checking build, libmoe_mxfp4_bounds.so), then switch back."""
    global _lib
    other = load_library(path)
    prev = lib()
    with _lock:
        _lib = other
    try:
        yield other
    finally:
        with _lock:
            _lib = prev


def load_library(path: str):
    """Load a build of the library and declare its functions' argument types."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing")
    L = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    dp = ctypes.POINTER(moe_dims)
    L.moe_mxfp4_codes_bytes.argtypes = [i32, i32, i32]
    L.moe_mxfp4_codes_bytes.restype = sz
    L.moe_mxfp4_scales_bytes.argtypes = [i32, i32, i32]
    L.moe_mxfp4_scales_bytes.restype = sz
    L.moe_mxfp4_quantize.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    L.moe_mxfp4_quantize.restype = ctypes.c_int
    L.moe_workspace_bytes.argtypes = [dp, i32]
    L.moe_workspace_bytes.restype = sz
    L.moe_route.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_route.restype = ctypes.c_int
    L.moe_forward.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_forward.restype = ctypes.c_int
    L.moe_forward_timed.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                    vp, i32]
    L.moe_forward_timed.restype = ctypes.c_int
    L.moe_resolve_path.argtypes = [dp, i32]
    L.moe_resolve_path.restype = i32
    L.moe_workspace_layout.argtypes = [dp, i32, vp]
    L.moe_workspace_layout.restype = ctypes.c_int
    L.moe_device_status.argtypes = [vp, vp]
    L.moe_device_status.restype = ctypes.c_int
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_forward_partial.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_forward_partial.restype = ctypes.c_int
    L.moe_forward_norm.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                   vp, sz, vp]
    L.moe_forward_norm.restype = ctypes.c_int
    L.moe_residual_norm.argtypes = [i32, i32, vp, vp, vp, ctypes.c_float, vp, vp, vp]
    L.moe_residual_norm.restype = ctypes.c_int
    L.moe_forward_no_alloc.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_forward_no_alloc.restype = ctypes.c_int
    L.moe_forward_host.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i32, vp, vp, vp]
    L.moe_forward_host.restype = ctypes.c_int
    L.moe_host_chunk_tokens.argtypes = [dp, i32]
    L.moe_host_chunk_tokens.restype = i32
    L.moe_debug_inject_timeout.argtypes = [i32]
    L.moe_debug_inject_timeout.restype = None
    L.moe_last_launch_count.argtypes = []
    L.moe_last_launch_count.restype = i32
    return L


def header_functions() -> list[str]:
    """Names of the functions include/moe_mxfp4.h declares."""
    txt = open(HEADER_PATH).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", txt)))


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(st: int, what: str):
    if st != MOE_OK:
        raise MoeError(st, what)


def _need(t: torch.Tensor, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name}: a CUDA tensor is required")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def moe_mxfp4_codes_bytes(E: int, N: int, K: int) -> int:
    return lib().moe_mxfp4_codes_bytes(E, N, K)


def moe_mxfp4_scales_bytes(E: int, N: int, K: int) -> int:
    return lib().moe_mxfp4_scales_bytes(E, N, K)


def kpad128(K: int) -> int:
    return (K + 127) // 128 * 128


def mxfp4_shapes(E: int, N: int, K: int):
    """Tensor shapes of the library's MXFP4 storage (see include/moe_mxfp4.h):
    codes [E, NT, KC, 128, 64], scales [E, NT, KC, 512] (uint8), NT = ceil(N/128), KC = ceil(K/128)."""
    NT, KC = (N + 127) // 128, kpad128(K) // 128
    return (E, NT, KC, 128, 64), (E, NT, KC, 512)


def moe_mxfp4_quantize(w: torch.Tensor, codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                       role: int | str = MOE_WEIGHT_PLAIN, status_word: torch.Tensor | None = None, stream=None):
    """fp32 weights [E, N, K] -> (codes, scales) in the library's MXFP4 storage.
    role: "gate_up" for W1 [E, 2I, d] (gate rows then up rows), "down"/"plain" otherwise."""
    if isinstance(role, str):
        role = ROLES[role]
    if w.dim() == 2:
        w = w.unsqueeze(0)
    _need(w, torch.float32, "w")
    E, N, K = w.shape
    cs, ss = mxfp4_shapes(E, N, K)
    if codes is None:
        codes = torch.empty(cs, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(ss, dtype=torch.uint8, device=w.device)
    if codes.numel() != moe_mxfp4_codes_bytes(E, N, K) or scales.numel() != moe_mxfp4_scales_bytes(E, N, K):
        raise ValueError("codes / scales have the wrong size")
    _check(lib().moe_mxfp4_quantize(_ptr(w), E, N, K, role, _ptr(codes), _ptr(scales), _ptr(status_word),
                                    _stream(stream)), "moe_mxfp4_quantize")
    return codes, scales


def moe_workspace_bytes(dims: moe_dims, T: int) -> int:
    return lib().moe_workspace_bytes(ctypes.byref(dims), T)


def new_workspace(dims: moe_dims, T: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace (its status word starts clear)."""
    n = moe_workspace_bytes(dims, T)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_route(dims: moe_dims, x, norm_w, router_w, router_b, ws, stream=None):
    """-> dict(topk_idx [T,k] int32, topk_w [T,k] f32, counts [E], offsets [E+1], perm [T*k])."""
    T = x.shape[0]
    _need(x, torch.bfloat16, "x")
    dev = x.device
    k, E = dims.top_k, dims.E
    out = dict(topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
               topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               perm=torch.empty(T * k, dtype=torch.int32, device=dev))
    _check(lib().moe_route(ctypes.byref(dims), T, _ptr(x), _ptr(norm_w), _ptr(router_w), _ptr(router_b),
                           _ptr(out["topk_idx"]), _ptr(out["topk_w"]), _ptr(out["counts"]), _ptr(out["offsets"]),
                           _ptr(out["perm"]), _ptr(ws), ws.numel(), _stream(stream)), "moe_route")
    return out


def moe_forward(dims: moe_dims, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, ws,
                y=None, want_routing=False, stream=None):
    """y [T, d] bf16 = x + MoE(RMSNorm(x)); with want_routing also (topk_idx, topk_w, counts)."""
    T = x.shape[0]
    _need(x, torch.bfloat16, "x")
    dev = x.device
    if y is None:
        y = torch.empty_like(x)
    r = None
    if want_routing:
        r = dict(topk_idx=torch.empty((T, dims.top_k), dtype=torch.int32, device=dev),
                 topk_w=torch.empty((T, dims.top_k), dtype=torch.float32, device=dev),
                 counts=torch.empty(dims.E, dtype=torch.int32, device=dev))
    _check(lib().moe_forward(ctypes.byref(dims), T, _ptr(x), _ptr(norm_w), _ptr(router_w), _ptr(router_b),
                             _ptr(w1_codes), _ptr(w1_scales), _ptr(w2_codes), _ptr(w2_scales), _ptr(y),
                             _ptr(r["topk_idx"]) if r else None, _ptr(r["topk_w"]) if r else None,
                             _ptr(r["counts"]) if r else None, _ptr(ws), ws.numel(), _stream(stream)),
           "moe_forward")
    return (y, r) if want_routing else y


def moe_host_chunk_tokens(dims: moe_dims, T: int) -> int:
    """Tokens per chunk moe_forward_host takes when left to choose (T for one chunk)."""
    n = lib().moe_host_chunk_tokens(ctypes.byref(dims), T)
    if n < 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_host_chunk_tokens")
    return n


def _need_host(t: torch.Tensor, name, shape):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name}: a host (CPU) tensor is required")
    if t.dtype != torch.bfloat16 or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: a contiguous bf16 tensor of shape {tuple(shape)} is required")


def moe_forward_host(dims: moe_dims, x_host, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales,
                     ws, x_dev, y_dev, y_host=None, chunk_tokens=0, h2d_stream=None, d2h_stream=None, stream=None):
    """y_host [T, d] bf16 (host, page-locked) = x_host + MoE(RMSNorm(x_host)), staged through the
    device buffers x_dev / y_dev [T, d] in chunks whose copies overlap the layer (h2d_stream and
    d2h_stream carry the copies; None runs them on `stream`).  Returns y_host once enqueued:
    synchronize `stream` before reading it."""
    T, d = x_host.shape
    _need_host(x_host, "x_host", (T, d))
    if y_host is None:
        y_host = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
    _need_host(y_host, "y_host", (T, d))
    _need(x_dev, torch.bfloat16, "x_dev", (T, d))
    _need(y_dev, torch.bfloat16, "y_dev", (T, d))
    hs = ctypes.c_void_p(h2d_stream.cuda_stream) if h2d_stream is not None else None
    ds = ctypes.c_void_p(d2h_stream.cuda_stream) if d2h_stream is not None else None
    _check(lib().moe_forward_host(ctypes.byref(dims), T, _ptr(x_host), _ptr(y_host), _ptr(x_dev), _ptr(y_dev),
                                  _ptr(norm_w), _ptr(router_w), _ptr(router_b), _ptr(w1_codes), _ptr(w1_scales),
                                  _ptr(w2_codes), _ptr(w2_scales), _ptr(ws), ws.numel(), int(chunk_tokens),
                                  _stream(stream), hs, ds), "moe_forward_host")
    return y_host


def moe_forward_partial(dims: moe_dims, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales,
                        ws, y_partial=None, want_routing=False, stream=None):
    """One slice of the intermediate features (weights of the slice, dims.I = its width):
    y_partial [T, d] fp32 = the slice's share of the expert mix, without the residual."""
    T = x.shape[0]
    _need(x, torch.bfloat16, "x")
    dev = x.device
    if y_partial is None:
        y_partial = torch.empty((T, dims.d), dtype=torch.float32, device=dev)
    r = None
    if want_routing:
        r = dict(topk_idx=torch.empty((T, dims.top_k), dtype=torch.int32, device=dev),
                 topk_w=torch.empty((T, dims.top_k), dtype=torch.float32, device=dev),
                 counts=torch.empty(dims.E, dtype=torch.int32, device=dev))
    _check(lib().moe_forward_partial(ctypes.byref(dims), T, _ptr(x), _ptr(norm_w), _ptr(router_w), _ptr(router_b),
                                     _ptr(w1_codes), _ptr(w1_scales), _ptr(w2_codes), _ptr(w2_scales), _ptr(y_partial),
                                     _ptr(r["topk_idx"]) if r else None, _ptr(r["topk_w"]) if r else None,
                                     _ptr(r["counts"]) if r else None, _ptr(ws), ws.numel(), _stream(stream)),
           "moe_forward_partial")
    return (y_partial, r) if want_routing else y_partial


def moe_forward_norm(dims: moe_dims, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, ws,
                     next_norm_w, next_eps=1e-5, y=None, y_norm=None, stream=None):
    """(y, y_norm): the layer's output and the next block's RMSNorm of it, in one pass."""
    _need(x, torch.bfloat16, "x")
    _need(next_norm_w, torch.float32, "next_norm_w", (dims.d,))
    y = torch.empty_like(x) if y is None else y
    y_norm = torch.empty_like(x) if y_norm is None else y_norm
    _check(lib().moe_forward_norm(ctypes.byref(dims), x.shape[0], _ptr(x), _ptr(norm_w), _ptr(router_w),
                                  _ptr(router_b), _ptr(w1_codes), _ptr(w1_scales), _ptr(w2_codes), _ptr(w2_scales),
                                  _ptr(next_norm_w), float(next_eps), _ptr(y), _ptr(y_norm), _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_forward_norm")
    return y, y_norm


def moe_residual_norm(x, s, norm_w=None, eps=1e-5, y=None, y_norm=None, stream=None):
    """y = bf16(x + s) for fp32 s [T, d]; with norm_w also y_norm = bf16(RMSNorm(y) * norm_w)."""
    _need(x, torch.bfloat16, "x")
    _need(s, torch.float32, "s", tuple(x.shape))
    T, d = x.shape
    y = torch.empty_like(x) if y is None else y
    if norm_w is not None and y_norm is None:
        y_norm = torch.empty_like(x)
    _check(lib().moe_residual_norm(T, d, _ptr(x), _ptr(s), _ptr(norm_w), float(eps), _ptr(y),
                                   _ptr(y_norm) if norm_w is not None else None, _stream(stream)),
           "moe_residual_norm")
    return (y, y_norm) if norm_w is not None else y


def intermediate_slices(I: int, G: int) -> list[tuple[int, int]]:
    """[i0, i1) of G slices of the intermediate features, each a multiple of 64 wide (the
    64-feature blocks dealt out as evenly as they go: 2880 = 45 blocks -> 23 + 22 for G = 2)."""
    if I % 64 or G < 1 or G > I // 64:
        raise ValueError(f"cannot cut I = {I} into {G} slices of whole 64-feature blocks")
    nb = I // 64
    out, b0 = [], 0
    for g in range(G):
        nbg = nb // G + (1 if g < nb % G else 0)
        out.append((64 * b0, 64 * (b0 + nbg)))
        b0 += nbg
    return out


WS_FIELDS = ("status", "counts", "offsets", "ntiles", "tile_base", "tiles", "topk_idx", "topk_w", "perm", "inv",
             "w_sorted", "xq", "xsf", "bpx", "bph", "ys", "total")


def moe_workspace_layout(dims: moe_dims, T: int) -> dict:
    """Byte offsets of the workspace sub-buffers (for tests and debugging)."""
    arr = (ctypes.c_size_t * len(WS_FIELDS))()
    _check(lib().moe_workspace_layout(ctypes.byref(dims), T, arr), "moe_workspace_layout")
    return dict(zip(WS_FIELDS, list(arr)))


def workspace_view(ws: torch.Tensor, dims: moe_dims, T: int, field: str, dtype, shape) -> torch.Tensor:
    """A typed view of one workspace sub-buffer."""
    off = moe_workspace_layout(dims, T)[field]
    n = 1
    for s_ in shape:
        n *= s_
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(*shape)


def moe_forward_timed(dims: moe_dims, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, ws,
                      y=None, events=None, stream=None):
    """moe_forward that records ``events`` (torch.cuda.Event, timing enabled) around each kernel:
    event 2i before kernel i and 2i+1 after it (kernels: route, group, pack, gate_up, down, combine;
    small batches: route with the grouping, pack, gate_up, down, combine)."""
    _need(x, torch.bfloat16, "x")
    if y is None:
        y = torch.empty_like(x)
    arr, n = None, 0
    if events:
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        n = len(events)
    _check(lib().moe_forward_timed(ctypes.byref(dims), x.shape[0], _ptr(x), _ptr(norm_w), _ptr(router_w),
                                   _ptr(router_b), _ptr(w1_codes), _ptr(w1_scales), _ptr(w2_codes), _ptr(w2_scales),
                                   _ptr(y), None, None, None, _ptr(ws), ws.numel(), _stream(stream), arr, n),
           "moe_forward_timed")
    return y


PATH_NAMES = {v: k for k, v in PATHS.items()}


def resolved_path(dims: moe_dims, T: int) -> str:
    """The path moe_forward takes for these dims and T (resolves MOE_PATH_AUTO)."""
    return PATH_NAMES[lib().moe_resolve_path(ctypes.byref(dims), T)]


def moe_device_status(ws: torch.Tensor, stream=None) -> int:
    return lib().moe_device_status(_ptr(ws), _stream(stream))


def last_launch_count() -> int:
    return lib().moe_last_launch_count()


def moe_forward_no_alloc(dims: moe_dims, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales,
                         y=None, status_out=None, stream=None):
    """moe_forward without a workspace, for callers that cannot allocate device memory while
    they run (the library's fixed 16 MiB device scratch is used instead; see the header).
    ``y`` and ``status_out`` (int32 [1]) are caller buffers; this wrapper creates ``y`` with
    torch only when it is not given."""
    _need(x, torch.bfloat16, "x")
    if y is None:
        y = torch.empty_like(x)
    _check(lib().moe_forward_no_alloc(ctypes.byref(dims), x.shape[0], _ptr(x), _ptr(norm_w), _ptr(router_w),
                                      _ptr(router_b), _ptr(w1_codes), _ptr(w1_scales), _ptr(w2_codes),
                                      _ptr(w2_scales), _ptr(y), _ptr(status_out), _stream(stream)),
           "moe_forward_no_alloc")
    return y


def moe_debug_inject_timeout(enable: bool = True) -> None:
    """Test hook: the next tensor-core forward on this thread times out in one CTA (see the header)."""
    lib().moe_debug_inject_timeout(1 if enable else 0)
