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
#include <cuda_runtime.h>
#include <mutex>

#include "moe_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_no_alloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The array's name in host
// code is only a host-side handle; the address must come from cudaGetSymbolAddress,
// once per device, with that device current.
moe_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_forward_no_alloc(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                                const float* router_w, const float* router_b, const uint8_t* w1_codes,
                                const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                                uint16_t* y, int32_t* status_out, void* stream) {
  const size_t need = moe_workspace_bytes(dims, T);
  if (need == 0) return dims ? MOE_ERR_UNSUPPORTED_SHAPE : MOE_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  void* ws = nullptr;
  moe_status st = scratch_for_current_device(&ws);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, moe::kStatusBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  st = moe_forward(dims, T, x, norm_w, router_w, router_b, w1_codes, w1_scales, w2_codes, w2_scales, y, nullptr,
                   nullptr, nullptr, ws, kNoAllocScratchBytes, stream);
  if (st != MOE_OK) return st;
  if (status_out && cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
