// C-ABI front end: argument checks, workspace carve-up, path choice, launches.
// Declarations and the contract of every entry point: include/moe_mxfp4.h.
#include <cuda_runtime.h>
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <vector>

#include "moe_internal.cuh"

namespace {

thread_local int32_t g_last_launches = 0;
thread_local int32_t g_inject_timeout = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Compute capability check, remembered per device (bit set = checked and sm_100).
std::atomic<uint64_t> g_device_ok{0};

moe_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (dev < 64 && (g_device_ok.load(std::memory_order_acquire) & bit)) return MOE_OK;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MOE_ERR_DEVICE;
  if (dev < 64) g_device_ok.fetch_or(bit, std::memory_order_release);
  return MOE_OK;
}

moe_status check_dims(const moe_dims* dm, int32_t T) {
  if (!dm || T < 0) return MOE_ERR_INVALID_ARG;
  if (dm->path < MOE_PATH_AUTO || dm->path > MOE_PATH_GEMM) return MOE_ERR_INVALID_ARG;
  if (dm->act_format != MOE_ACT_BF16 && dm->act_format != MOE_ACT_MXFP8 && dm->act_format != MOE_ACT_MXFP4)
    return MOE_ERR_INVALID_ARG;
  if (!(dm->rms_eps >= 0.f) || !std::isfinite(dm->rms_eps)) return MOE_ERR_INVALID_ARG;
  if (!(dm->swiglu_limit > 0.f) || !std::isfinite(dm->swiglu_limit)) return MOE_ERR_INVALID_ARG;
  if (dm->block != 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dm->d <= 0 || dm->I <= 0 || dm->d % 64 || dm->I % 64) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dm->d > (1 << 16) || dm->I > (1 << 16)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dm->E < 1 || dm->E > 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dm->top_k < 1 || dm->top_k > dm->E || dm->top_k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)T * dm->top_k > (int64_t(1) << 24)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

#ifndef MOE_GEMV_FUSE_COMBINE
#define MOE_GEMV_FUSE_COMBINE 0
#endif

int resolve_path(const moe_dims& dm, int32_t T) {
  if (dm.path != MOE_PATH_AUTO) return dm.path;
  // Few tokens per expert: stream the weights with narrow token tiles.
  const double per_expert = (double)T * dm.top_k / dm.E;
  return per_expert <= 24.0 ? MOE_PATH_GEMV : MOE_PATH_GEMM;
}

// Activation rows per token fed to the expert GEMMs: bf16 activations travel as two E4M3
// terms; MXFP8 as one E4M3 row, MXFP4 as one row of packed E2M1 codes.
int terms_of(const moe_dims& dm) { return dm.act_format == MOE_ACT_BF16 ? 2 : 1; }

moe::WsLayout layout_for(const moe_dims& dm, int32_t T) {
  const int path = resolve_path(dm, T), terms = terms_of(dm);
  return moe::ws_layout(dm, T, moe::expert_tile_tokens(path, terms), moe::expert_down_split(path), terms,
                        dm.act_format == MOE_ACT_MXFP4 ? 1 : 0);
}

moe_status prepare(const moe_dims* dm, int32_t T, const uint16_t* x, const float* norm_w, const float* router_w,
                   const float* router_b, void* ws, size_t ws_bytes, moe::FwdArgs& a, moe::WsLayout& L) {
  moe_status st = check_dims(dm, T);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;  // nothing to do; empty tensors may carry null pointers
  if (!x || !norm_w || !router_w || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(norm_w) || !aligned16(router_w) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (router_b && !aligned16(router_b)) return MOE_ERR_INVALID_ARG;
  L = layout_for(*dm, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  st = check_device();
  if (st != MOE_OK) return st;
  std::memset(&a, 0, sizeof(a));
  a.T = T;
  a.d = dm->d;
  a.I = dm->I;
  a.E = dm->E;
  a.k = dm->top_k;
  a.eps = dm->rms_eps;
  a.limit = dm->swiglu_limit;
  a.x = x;
  a.norm_w = norm_w;
  a.router_w = router_w;
  a.router_b = router_b;
  a.ws = moe::ws_pointers(ws, L, dm->E);
  return MOE_OK;
}

moe_status copy_out(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!dst) return MOE_OK;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Where a forward call writes the layer's output.
struct Outputs {
  uint16_t* y = nullptr;               // bf16 [T][d]: x + the expert mix
  float* y_partial = nullptr;          // fp32 [T][d]: the expert mix alone (instead of y)
  const float* next_norm_w = nullptr;  // with y_norm: the next block's RMSNorm of y
  float next_eps = 0.f;
  uint16_t* y_norm = nullptr;
  int32_t* topk_idx = nullptr;
  float* topk_w = nullptr;
  int32_t* counts = nullptr;
};

moe_status forward_impl(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                        const float* router_w, const float* router_b, const uint8_t* w1_codes,
                        const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                        const Outputs& out, void* ws, size_t ws_bytes, void* stream, void* const* events,
                        int32_t n_events) {
  g_last_launches = 0;
  if (n_events < 0 || (n_events > 0 && !events)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_dims(dims, T);
  if (st != MOE_OK) return st;
  if (T > 0) {  // (argument errors come before any device query)
    if (!w1_codes || !w1_scales || !w2_codes || !w2_scales) return MOE_ERR_INVALID_ARG;
    if (!aligned32(w1_codes) || !aligned16(w1_scales) || !aligned32(w2_codes) || !aligned16(w2_scales))
      return MOE_ERR_INVALID_ARG;
    void* const dst = out.y_partial ? static_cast<void*>(out.y_partial) : static_cast<void*>(out.y);
    if (!dst || !aligned16(dst) || (const void*)dst == (const void*)x) return MOE_ERR_INVALID_ARG;
    if (out.next_norm_w) {
      if (!out.y_norm || !aligned16(out.next_norm_w) || !aligned16(out.y_norm)) return MOE_ERR_INVALID_ARG;
      if ((void*)out.y_norm == (void*)out.y || (const void*)out.y_norm == (const void*)x) return MOE_ERR_INVALID_ARG;
      if (!(out.next_eps >= 0.f) || !std::isfinite(out.next_eps)) return MOE_ERR_INVALID_ARG;
    }
  }
  moe::FwdArgs a;
  moe::WsLayout L;
  st = prepare(dims, T, x, norm_w, router_w, router_b, ws, ws_bytes, a, L);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  a.w1c = w1_codes;
  a.w1s = w1_scales;
  a.w2c = w2_codes;
  a.w2s = w2_scales;
  a.y = out.y;
  a.y_partial = out.y_partial;
  a.next_norm_w = out.next_norm_w;
  a.next_eps = out.next_eps;
  a.y_norm = out.y_norm;
  a.stream = static_cast<cudaStream_t>(stream);
  moe::EventRec rec;
  rec.events = events;
  rec.n = n_events;
  if (n_events > 0) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(a.stream, &cs) != cudaSuccess) return MOE_ERR_CUDA;
    rec.capturing = cs == cudaStreamCaptureStatusActive;
  }
  a.ev = &rec;
  a.inject_timeout = g_inject_timeout;
  g_inject_timeout = 0;
  const int path = resolve_path(*dims, T);
  // Small-batch path: fewer, fused kernels (routing + grouping + tile scales; down + combine).
  // The next block's RMSNorm needs whole rows, which the separate combine pass holds.
  a.fuse_group = (path == MOE_PATH_GEMV && T <= moe::kFusedGroupMaxT) ? 1 : 0;
  // The combine runs as its own pass after the down GEMM, so that the down GEMM can split
  // its reduction axis as finely as balances the CTAs without a combining epilogue per
  // split.  MOE_GEMV_FUSE_COMBINE=1 builds the fused form (the last writer of each token's
  // 128 columns combines).
  a.fuse_combine = (MOE_GEMV_FUSE_COMBINE && path == MOE_PATH_GEMV && !a.next_norm_w) ? 1 : 0;
  // Overlap each kernel's launch and prologue with its predecessor, except when per-kernel
  // events are recorded between the kernels.
  a.pdl = (n_events == 0) ? 1 : 0;
  int n = moe::launch_route(a);
  if (n < 0) return MOE_ERR_CUDA;
  const int ne = moe::launch_experts(a);
  if (ne < 0) return MOE_ERR_CUDA;
  n += ne;
  if (!a.fuse_combine) {
    const int nc = moe::launch_combine(a);
    if (nc < 0) return MOE_ERR_CUDA;
    n += nc;
  }
  const size_t P = (size_t)T * dims->top_k;
  if ((st = copy_out(out.topk_idx, a.ws.topk_idx, 4 * P, a.stream)) != MOE_OK) return st;
  if ((st = copy_out(out.topk_w, a.ws.topk_w, 4 * P, a.stream)) != MOE_OK) return st;
  if ((st = copy_out(out.counts, a.ws.counts, 4 * (size_t)dims->E, a.stream)) != MOE_OK) return st;
  g_last_launches = n;
  return MOE_OK;
}

// Tokens per chunk of moe_forward_host when the caller leaves the choice to the library.
// A chunk's copies in and out overlap the layer of its neighbours, but every chunk streams
// the expert weights once more and fills its token tiles less: one chunk on the small-batch
// path and below 4096 tokens (copies of a few MB), else two to four chunks of at least 2048
// tokens.
int32_t host_chunk(const moe_dims& dm, int32_t T) {
  if (T < 4096 || resolve_path(dm, T) == MOE_PATH_GEMV) return T;
  const int32_t n = std::min<int32_t>(4, T / 2048);
  return (T + n - 1) / n;
}

// Events for the copy / layer overlap of moe_forward_host, per device and host thread
// (timing disabled; reused call after call: a wait takes the event's state at the time it
// is enqueued).
struct HostEvents {
  std::vector<cudaEvent_t> ev[64];
  ~HostEvents() {
    for (auto& v : ev)
      for (cudaEvent_t e : v) cudaEventDestroy(e);
  }
  cudaEvent_t get(int dev, size_t i) {
    if (dev < 0 || dev >= 64) return nullptr;
    std::vector<cudaEvent_t>& v = ev[dev];
    while (v.size() <= i) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
      v.push_back(e);
    }
    return v[i];
  }
};
thread_local HostEvents g_host_events;

}  // namespace

namespace moe {
moe_status validate_dims(const moe_dims* dims, int32_t T) { return check_dims(dims, T); }
}  // namespace moe

extern "C" {

size_t moe_mxfp4_codes_bytes(int32_t E, int32_t N, int32_t K) {
  if (E <= 0 || N <= 0 || K <= 0) return 0;
  return (size_t)E * (size_t)((N + 127) / 128) * (size_t)(moe::kpad128(K) / moe::kKChunk) * moe::kCodeBlockBytes;
}

size_t moe_mxfp4_scales_bytes(int32_t E, int32_t N, int32_t K) {
  if (E <= 0 || N <= 0 || K <= 0) return 0;
  return (size_t)E * (size_t)((N + 127) / 128) * (size_t)(moe::kpad128(K) / moe::kKChunk) * moe::kSfGroupBytes;
}

moe_status moe_mxfp4_quantize(const float* w, int32_t E, int32_t N, int32_t K, int32_t role, uint8_t* codes,
                              uint8_t* scales, int32_t* status_word, void* stream) {
  g_last_launches = 0;
  if (!w || !codes || !scales || E <= 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (role != MOE_WEIGHT_PLAIN && role != MOE_WEIGHT_GATE_UP) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned32(codes) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
  if (K % 64 || N % 64) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (role == MOE_WEIGHT_GATE_UP && (N / 2) % 64) return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_status st = check_device();
  if (st != MOE_OK) return st;
  const int n = moe::launch_quantize(w, E, N, K, role, codes, scales, status_word, static_cast<cudaStream_t>(stream));
  if (n < 0) return MOE_ERR_CUDA;
  g_last_launches = n;
  return MOE_OK;
}

size_t moe_workspace_bytes(const moe_dims* dims, int32_t T) {
  if (check_dims(dims, T) != MOE_OK) return 0;
  return layout_for(*dims, T).total;
}

moe_status moe_route(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                     const float* router_w, const float* router_b, int32_t* topk_idx, float* topk_w,
                     int32_t* counts, int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  g_last_launches = 0;
  moe::FwdArgs a;
  moe::WsLayout L;
  moe_status st = prepare(dims, T, x, norm_w, router_w, router_b, ws, ws_bytes, a, L);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  a.stream = static_cast<cudaStream_t>(stream);
  const int n = moe::launch_route(a);
  if (n < 0) return MOE_ERR_CUDA;
  const size_t P = (size_t)T * dims->top_k;
  if ((st = copy_out(topk_idx, a.ws.topk_idx, 4 * P, a.stream)) != MOE_OK) return st;
  if ((st = copy_out(topk_w, a.ws.topk_w, 4 * P, a.stream)) != MOE_OK) return st;
  if ((st = copy_out(counts, a.ws.counts, 4 * (size_t)dims->E, a.stream)) != MOE_OK) return st;
  if ((st = copy_out(offsets, a.ws.offsets, 4 * (size_t)(dims->E + 1), a.stream)) != MOE_OK) return st;
  if ((st = copy_out(perm, a.ws.perm, 4 * P, a.stream)) != MOE_OK) return st;
  g_last_launches = n;
  return MOE_OK;
}

moe_status moe_forward(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                       const float* router_w, const float* router_b, const uint8_t* w1_codes,
                       const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales, uint16_t* y,
                       int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                       void* stream) {
  return moe_forward_timed(dims, T, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, y,
                           topk_idx_out, topk_w_out, counts_out, ws, ws_bytes, stream, nullptr, 0);
}

moe_status moe_forward_timed(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                             const float* router_w, const float* router_b, const uint8_t* w1_codes,
                             const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                             uint16_t* y, int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, void* ws,
                             size_t ws_bytes, void* stream, void* const* events, int32_t n_events) {
  Outputs out;
  out.y = y;
  out.topk_idx = topk_idx_out;
  out.topk_w = topk_w_out;
  out.counts = counts_out;
  return forward_impl(dims, T, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, out, ws,
                      ws_bytes, stream, events, n_events);
}

moe_status moe_forward_partial(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                               const float* router_w, const float* router_b, const uint8_t* w1_codes,
                               const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                               float* y_partial, int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out,
                               void* ws, size_t ws_bytes, void* stream) {
  Outputs out;
  out.y_partial = y_partial;
  out.topk_idx = topk_idx_out;
  out.topk_w = topk_w_out;
  out.counts = counts_out;
  return forward_impl(dims, T, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, out, ws,
                      ws_bytes, stream, nullptr, 0);
}

moe_status moe_forward_norm(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                            const float* router_w, const float* router_b, const uint8_t* w1_codes,
                            const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                            const float* next_norm_w, float next_eps, uint16_t* y, uint16_t* y_norm, void* ws,
                            size_t ws_bytes, void* stream) {
  Outputs out;
  out.y = y;
  out.next_norm_w = next_norm_w;
  out.next_eps = next_eps;
  out.y_norm = y_norm;
  return forward_impl(dims, T, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, out, ws,
                      ws_bytes, stream, nullptr, 0);
}

moe_status moe_residual_norm(int32_t T, int32_t d, const uint16_t* x, const float* s, const float* norm_w,
                             float eps, uint16_t* y, uint16_t* y_norm, void* stream) {
  g_last_launches = 0;
  if (T < 0 || d <= 0 || d % 64 || d > (1 << 16)) return T < 0 || d <= 0 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !s || !y || !aligned16(x) || !aligned16(s) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if ((const void*)y == (const void*)x) return MOE_ERR_INVALID_ARG;
  if (norm_w) {
    if (!y_norm || !aligned16(norm_w) || !aligned16(y_norm) || y_norm == y || (const void*)y_norm == (const void*)x)
      return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return MOE_ERR_INVALID_ARG;
  }
  const moe_status st = check_device();
  if (st != MOE_OK) return st;
  if (moe::launch_residual_norm(T, d, x, s, norm_w, eps, y, norm_w ? y_norm : nullptr,
                                static_cast<cudaStream_t>(stream)) < 0)
    return MOE_ERR_CUDA;
  g_last_launches = 1;
  return MOE_OK;
}

int32_t moe_host_chunk_tokens(const moe_dims* dims, int32_t T) {
  if (check_dims(dims, T) != MOE_OK) return -1;
  return host_chunk(*dims, T);
}

moe_status moe_forward_host(const moe_dims* dims, int32_t T, const uint16_t* x_host, uint16_t* y_host,
                            uint16_t* x_dev, uint16_t* y_dev, const float* norm_w, const float* router_w,
                            const float* router_b, const uint8_t* w1_codes, const uint8_t* w1_scales,
                            const uint8_t* w2_codes, const uint8_t* w2_scales, void* ws, size_t ws_bytes,
                            int32_t chunk_tokens, void* stream, void* h2d_stream, void* d2h_stream) {
  g_last_launches = 0;
  moe_status st = check_dims(dims, T);
  if (st != MOE_OK) return st;
  if (chunk_tokens < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  // Every argument check of the chunks' forward calls, made before anything is enqueued.
  if (!x_host || !y_host || !x_dev || !y_dev || !norm_w || !router_w || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_dev) || !aligned16(y_dev) || !aligned16(norm_w) || !aligned16(router_w) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  if ((void*)x_dev == (void*)y_dev || (router_b && !aligned16(router_b))) return MOE_ERR_INVALID_ARG;
  if (!w1_codes || !w1_scales || !w2_codes || !w2_scales) return MOE_ERR_INVALID_ARG;
  if (!aligned32(w1_codes) || !aligned16(w1_scales) || !aligned32(w2_codes) || !aligned16(w2_scales))
    return MOE_ERR_INVALID_ARG;
  const int32_t chunk = chunk_tokens > 0 ? std::min(chunk_tokens, T) : host_chunk(*dims, T);
  const int32_t n = (T + chunk - 1) / chunk;
  const int32_t last = T - (n - 1) * chunk;
  if (ws_bytes < layout_for(*dims, chunk).total || ws_bytes < layout_for(*dims, last).total)
    return MOE_ERR_WORKSPACE;
  if ((st = check_device()) != MOE_OK) return st;

  // One chunk: copy in, layer and copy out in order on `stream`.  Several: the copies in on
  // h2d_stream, the layers on `stream`, the copies out on d2h_stream, ordered by events.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t sh = (n > 1 && h2d_stream) ? static_cast<cudaStream_t>(h2d_stream) : s;
  cudaStream_t sd = (n > 1 && d2h_stream) ? static_cast<cudaStream_t>(d2h_stream) : s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  // events: 0 fork, 1 join, 2 + 2c chunk c copied in, 3 + 2c chunk c's layer done
  if (!g_host_events.get(dev, 2 * (size_t)n + 1)) return MOE_ERR_CUDA;
  auto ev = [&](size_t i) { return g_host_events.get(dev, i); };
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  const size_t d = (size_t)dims->d, row_bytes = d * sizeof(uint16_t);
  auto rows_of = [&](int32_t c) { return c == n - 1 ? last : chunk; };

  // fork: the copies in wait for the work `stream` holds (which may still read x_dev)
  if (sh != s && !(ok(cudaEventRecord(ev(0), s)) && ok(cudaStreamWaitEvent(sh, ev(0), 0)))) return MOE_ERR_CUDA;
  for (int32_t c = 0; c < n; ++c) {
    const size_t off = (size_t)c * chunk * d;
    if (!ok(cudaMemcpyAsync(x_dev + off, x_host + off, rows_of(c) * row_bytes, cudaMemcpyHostToDevice, sh)))
      return MOE_ERR_CUDA;
    if (sh != s && !ok(cudaEventRecord(ev(2 + 2 * (size_t)c), sh))) return MOE_ERR_CUDA;
  }
  int32_t launches = 0;
  for (int32_t c = 0; c < n; ++c) {
    const size_t off = (size_t)c * chunk * d;
    if (sh != s && !ok(cudaStreamWaitEvent(s, ev(2 + 2 * (size_t)c), 0))) return MOE_ERR_CUDA;
    Outputs out;
    out.y = y_dev + off;
    st = forward_impl(dims, rows_of(c), x_dev + off, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes,
                      w2_scales, out, ws, ws_bytes, stream, nullptr, 0);
    if (st != MOE_OK) return st;
    launches += g_last_launches;
    if (sd != s && !(ok(cudaEventRecord(ev(3 + 2 * (size_t)c), s)) && ok(cudaStreamWaitEvent(sd, ev(3 + 2 * (size_t)c), 0))))
      return MOE_ERR_CUDA;
    if (!ok(cudaMemcpyAsync(y_host + off, y_dev + off, rows_of(c) * row_bytes, cudaMemcpyDeviceToHost, sd)))
      return MOE_ERR_CUDA;
  }
  // join: `stream` waits for the last copy out (the copies in were waited for chunk by chunk)
  if (sd != s && !(ok(cudaEventRecord(ev(1), sd)) && ok(cudaStreamWaitEvent(s, ev(1), 0)))) return MOE_ERR_CUDA;
  g_last_launches = launches;
  return MOE_OK;
}

int32_t moe_resolve_path(const moe_dims* dims, int32_t T) {
  if (check_dims(dims, T) != MOE_OK) return -1;
  return resolve_path(*dims, T);
}

moe_status moe_workspace_layout(const moe_dims* dims, int32_t T, size_t* offsets) {
  if (!offsets) return MOE_ERR_INVALID_ARG;
  const moe_status st = check_dims(dims, T);
  if (st != MOE_OK) return st;
  const moe::WsLayout L = layout_for(*dims, T);
  const size_t v[MOE_WS_FIELDS] = {L.status, L.counts, L.offsets,  L.ntiles, L.tile_base, L.tiles,
                                   L.topk_idx, L.topk_w, L.perm,   L.inv,      L.w_sorted, L.xq,
                                   L.xsf,    L.bpx,    L.bph,      L.ys,     L.total};
  for (int i = 0; i < MOE_WS_FIELDS; ++i) offsets[i] = v[i];
  return MOE_OK;
}

moe_status moe_device_status(void* ws, void* stream) {
  if (!ws || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0) {
    const int32_t zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return static_cast<moe_status>(v);
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_NONFINITE: return "non-finite value";
    case MOE_ERR_BOUNDS: return "store outside its buffer (bounds-checking build)";
    case MOE_ERR_DEVICE: return "device is not sm_100";
  }
  return "unknown status";
}

int32_t moe_last_launch_count(void) { return g_last_launches; }

void moe_debug_inject_timeout(int32_t enable) { g_inject_timeout = enable ? 1 : 0; }

}  // extern "C"
