// Internal declarations shared by the kernels and the C-ABI front end.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "moe_mxfp4.h"

namespace moe {

constexpr int kStatusBytes = 256;
constexpr int kMinTileTokens = 16;  // smallest token tile of any path (sizes the tile list)

// Token tile of the grouped expert kernels: rows [row0, row0 + rows) of the
// expert-sorted pair list, all belonging to expert `e`.
struct Tile {
  int32_t e;
  int32_t row0;
  int32_t rows;
  int32_t pad;
};

// Carve-up of the caller's workspace (byte offsets, 256-byte aligned).
struct WsLayout {
  size_t status;    // int32 device status word (first device error wins)
  size_t counts;    // int32 [E] expert histogram, then int32 [4] (routing ticket), then int32
                    // [T * ceil(d/128)] combine arrivals; cleared at the start of every call
  size_t offsets;   // int32 [E+1]
  size_t ntiles;    // int32 [4]: number of token tiles
  size_t tiles;     // Tile [max_tiles]
  size_t topk_idx;  // int32 [T*k]
  size_t topk_w;    // f32 [T*k]
  size_t perm;      // int32 [P]   sorted position -> t*k + slot
  size_t inv;       // int32 [P]   t*k + slot -> sorted position
  size_t w_sorted;  // f32 [P]     routing weight of each sorted pair
  size_t xe;        // f16 [T][d]  bf16(RMSNorm(x)) held as f16
  size_t xs;        // f16 [P][d]  xe gathered in sorted pair order
  size_t h;         // f16 [P][I]  SwiGLU output (bf16 values) in sorted order
  size_t ys;        // f32 [P][d]  routing-weighted expert outputs, sorted order
  size_t total;
  int64_t max_tiles;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline WsLayout ws_layout(const moe_dims& dm, int64_t T) {
  WsLayout L{};
  const int64_t P = T * dm.top_k;
  L.max_tiles = (P + kMinTileTokens - 1) / kMinTileTokens + dm.E;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.status = take(kStatusBytes);
  L.counts = take(4 * ((size_t)dm.E + 4 + (size_t)T * ((dm.d + 127) / 128)));
  L.offsets = take(4 * (size_t)(dm.E + 1));
  L.ntiles = take(16);
  L.tiles = take(sizeof(Tile) * (size_t)L.max_tiles);
  L.topk_idx = take(4 * (size_t)P);
  L.topk_w = take(4 * (size_t)P);
  L.perm = take(4 * (size_t)P);
  L.inv = take(4 * (size_t)P);
  L.w_sorted = take(4 * (size_t)P);
  L.xe = take(2 * (size_t)T * dm.d);
  L.xs = take(2 * (size_t)P * dm.d);
  L.h = take(2 * (size_t)P * dm.I);
  L.ys = take(4 * (size_t)P * dm.d);
  L.total = o;
  return L;
}

// Pointers into one workspace.
struct Ws {
  int32_t* status;
  int32_t* counts;
  int32_t* ticket;     // routing CTAs that finished (the last one builds the grouping)
  int32_t* arrivals;   // [T][ceil(d/128)] expert outputs written per (token, 128 columns)
  int32_t* offsets;
  int32_t* ntiles;
  Tile* tiles;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* perm;
  int32_t* inv;
  float* w_sorted;
  uint16_t* xe;
  uint16_t* xs;
  uint16_t* h;
  float* ys;
  int64_t max_tiles;
};

inline Ws ws_pointers(void* base, const WsLayout& L, int E) {
  char* b = static_cast<char*>(base);
  Ws w;
  w.status = reinterpret_cast<int32_t*>(b + L.status);
  w.counts = reinterpret_cast<int32_t*>(b + L.counts);
  w.offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  w.ntiles = reinterpret_cast<int32_t*>(b + L.ntiles);
  w.tiles = reinterpret_cast<Tile*>(b + L.tiles);
  w.topk_idx = reinterpret_cast<int32_t*>(b + L.topk_idx);
  w.topk_w = reinterpret_cast<float*>(b + L.topk_w);
  w.perm = reinterpret_cast<int32_t*>(b + L.perm);
  w.inv = reinterpret_cast<int32_t*>(b + L.inv);
  w.w_sorted = reinterpret_cast<float*>(b + L.w_sorted);
  w.xe = reinterpret_cast<uint16_t*>(b + L.xe);
  w.xs = reinterpret_cast<uint16_t*>(b + L.xs);
  w.h = reinterpret_cast<uint16_t*>(b + L.h);
  w.ys = reinterpret_cast<float*>(b + L.ys);
  w.ticket = w.counts + E;
  w.arrivals = w.counts + E + 4;
  w.max_tiles = L.max_tiles;
  return w;
}

// Optional per-kernel CUDA events supplied by the caller: event 2i is recorded just
// before the i-th kernel of a call and event 2i+1 just after it.
struct EventRec {
  void* const* events = nullptr;
  int n = 0;
  int next = 0;
  bool capturing = false;  // the stream is being captured: record as external graph nodes
};

inline void record_event(const EventRec& r, int i, cudaStream_t st) {
  cudaEvent_t e = static_cast<cudaEvent_t>(r.events[i]);
  if (r.capturing) cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else cudaEventRecord(e, st);
}

// Everything a forward launch needs.
struct FwdArgs {
  int32_t T, d, I, E, k;
  float eps, limit;
  const uint16_t* x;
  const float* norm_w;
  const float* router_w;
  const float* router_b;
  const uint8_t* w1c;
  const uint8_t* w1s;
  const uint8_t* w2c;
  const uint8_t* w2s;
  uint16_t* y;
  Ws ws;
  cudaStream_t stream;
  EventRec* ev;
  int32_t inject_timeout;  // test hook: withhold one pipeline arrival in the gate_up kernel
  int32_t fuse_group;      // small batches: the routing kernel also groups and gathers
  int32_t fuse_combine;    // the down kernel also adds the k expert outputs and the residual
  int32_t pdl;             // launch dependent kernels with programmatic stream serialization
};

// Programmatic dependent launch: a kernel launched with the attribute may start while
// its predecessor in the stream is still running; it calls pdl_wait() before touching
// anything the predecessor writes.  pdl_trigger() lets the successor start launching.
// Both are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                          Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

constexpr int kFusedGroupMaxT = 64;   // fused grouping: one CTA walks the tokens in order

inline void ev_before(const FwdArgs& a) {
  if (a.ev && a.ev->events && a.ev->next + 1 < a.ev->n) record_event(*a.ev, a.ev->next, a.stream);
}

inline void ev_after(const FwdArgs& a) {
  if (a.ev && a.ev->events && a.ev->next + 1 < a.ev->n) {
    record_event(*a.ev, a.ev->next + 1, a.stream);
    a.ev->next += 2;
  }
}

// ------------------------------------------------------------------ MXFP4 storage layout
// Weights [E][N][K] are stored in blocks of 64 rows x 64 k (N % 64 == 0, K % 64 == 0):
//   codes  [E][N/64][K/64][64 rows][32 bytes]   (one 2048-byte run per block)
//   scales [E][N/64][K/64][2][64]               (one 128-byte run per block)
// Row r of a block keeps its 64 codes as two 16-byte chunks (k 0..31 and k 32..63);
// chunk c sits at chunk position c ^ ((r >> 2) & 1), so that consecutive rows read by
// consecutive threads fall in different shared-memory banks.  Byte j of a chunk holds
// k = 2j (low nibble) and k = 2j + 1 (high nibble).  Scale byte (c, r) is the E8M0
// scale of row r, k = 32c .. 32c + 31 of the block.
constexpr int kBlkRows = 64;
constexpr int kBlkK = 64;
constexpr int kBlkCodeBytes = kBlkRows * kBlkK / 2;   // 2048
constexpr int kBlkScaleBytes = kBlkRows * kBlkK / 32; // 128

__host__ __device__ __forceinline__ int64_t mx_block_index(int64_t e, int64_t rb, int64_t ks, int64_t N, int64_t K) {
  return (e * (N / kBlkRows) + rb) * (K / kBlkK) + ks;
}

// Byte offset of the 16-byte code chunk holding k = 32*kb .. 32*kb+31 of row n.
__host__ __device__ __forceinline__ int64_t mx_code_chunk_offset(int64_t e, int64_t n, int64_t kb, int64_t N,
                                                                  int64_t K) {
  const int64_t r = n % kBlkRows, c = kb & 1;
  return mx_block_index(e, n / kBlkRows, kb >> 1, N, K) * kBlkCodeBytes + r * 32 + ((c ^ ((r >> 2) & 1)) << 4);
}

__host__ __device__ __forceinline__ int64_t mx_scale_offset(int64_t e, int64_t n, int64_t kb, int64_t N, int64_t K) {
  return mx_block_index(e, n / kBlkRows, kb >> 1, N, K) * kBlkScaleBytes + (kb & 1) * kBlkRows + n % kBlkRows;
}

// Record the first device-side error in the status word.
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// --------------------------------------------------------------------------- launchers
// Each returns the number of kernels it launched (>= 0) or -1 on a launch error.
int launch_quantize(const float* w, int64_t rows, int32_t N, int32_t K, int32_t E, uint8_t* codes,
                    uint8_t* scales, int32_t* status, cudaStream_t st);
int launch_route(const FwdArgs& a, int tile_tokens);   // norm + router + top-k + grouping + gather
int launch_combine(const FwdArgs& a);                  // y = x + sum_j ys[inv]
int launch_experts_simt(const FwdArgs& a);             // CUDA-core expert MLPs
int launch_experts_tc(const FwdArgs& a, int tile_tokens);  // tcgen05 expert MLPs
int tc_tile_tokens(int path);                          // token tile of a tensor-core path
int simt_tile_tokens();                                // token tile of the CUDA-core path

}  // namespace moe
