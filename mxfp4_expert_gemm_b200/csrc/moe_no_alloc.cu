// Forward entry point that allocates nothing: its scratch is a fixed-size array in
// the library's own device memory.
//
// Some callers cannot hand this library a workspace: code that runs where device
// allocation is not allowed or not available (inside an allocator or memory-pool
// callback, in a plugin host that only lends out its own tensors, or in a serving loop
// that forbids cudaMalloc and its implicit synchronization after start-up).  For them,
// moe_forward_no_alloc uses a file-scope __device__ array instead of a caller buffer.
//
// Every GPU that loads the library holds this array (kNoAllocScratchBytes) until the
// process exits.  All calls share it: calls that overlap on the GPU (different streams
// without ordering) race on it.  It keeps the previous call's contents; the parts that
// must start at zero (the device status word, the expert counters) are cleared on every
// call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

#include "moe_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxContexts = 64;

__device__ __align__(256) uint8_t g_no_alloc_scratch[kNoAllocScratchBytes];

// The array's address belongs to a CUDA context (the module is loaded once per context),
// so the lookup is remembered per current context.
struct ScratchEntry {
  CUcontext ctx;
  void* ptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxContexts] = {};
int g_scratch_n = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// Device address of the scratch array in the current context.  In host code the array's
// name is only a host-side handle; the address comes from cudaGetSymbolAddress with the
// context current.
moe_status scratch_for_current_context(void** out) {
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return MOE_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  for (int i = 0; ctx && i < g_scratch_n; ++i)
    if (g_scratch[i].ctx == ctx) {
      *out = g_scratch[i].ptr;
      return MOE_OK;
    }
  // (the lookup also makes the current device's primary context current when no context
  // was yet)
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
  if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return MOE_ERR_CUDA;
  if (g_scratch_n < kMaxContexts) g_scratch[g_scratch_n++] = {ctx, p};
  *out = p;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_forward_no_alloc(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                                const float* router_w, const float* router_b, const uint8_t* w1_codes,
                                const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                                uint16_t* y, int32_t* status_out, void* stream) {
  moe_status st = moe::validate_dims(dims, T);   // the same argument errors as moe_forward
  if (st != MOE_OK) return st;
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {   // nothing to compute; the call's status is OK
    if (status_out && cudaMemsetAsync(status_out, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (moe_workspace_bytes(dims, T) > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  void* ws = nullptr;
  st = scratch_for_current_context(&ws);
  if (st != MOE_OK) return st;
  if (cudaMemsetAsync(ws, 0, moe::kStatusBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  st = moe_forward(dims, T, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, y, nullptr,
                   nullptr, nullptr, ws, kNoAllocScratchBytes, stream);
  if (st != MOE_OK) return st;
  if (status_out && cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
