// Internal declarations shared by the kernels and the C-ABI front end.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstddef>
#include <cstdint>

#include "moe_mxfp4.h"

namespace moe {

constexpr int kStatusBytes = 256;
constexpr int kMinTileTokens = 8;   // smallest token tile of any path (sizes the tile list)
constexpr int kKChunk = 128;        // reduction-axis chunk: one TMA box row, one scale-factor group
constexpr int kSfGroupBytes = 512;  // scale factors of 128 rows x 4 blocks of 32

// Token tile of the grouped expert kernels: rows [row0, row0 + rows) of the
// expert-sorted pair list, all belonging to expert `e`.
struct Tile {
  int32_t e;
  int32_t row0;
  int32_t rows;
  int32_t pad;
};

__host__ __device__ __forceinline__ int64_t kpad128(int64_t K) { return (K + kKChunk - 1) / kKChunk * kKChunk; }

// Byte offset, within one 512-byte scale-factor group, of row r (of 128) and 32-block b
// (of 4): the layout the tensor cores' scale-factor copy (32 lanes x 16 bytes, repeated
// for the four lane quarters) expects.
__host__ __device__ __forceinline__ int sf_byte_in_group(int r, int b) {
  return (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

// A token tile feeds the MMA `rows` = terms * tile_tokens E4M3 rows (MMA columns): two
// per token (hi and lo term, bf16 activations) or one (MXFP8 activations); row n belongs
// to token n / terms.  Scale-factor groups: 128 rows each.
__host__ __device__ constexpr int sf_groups_of(int rows) { return (rows + 127) / 128; }

// Packed activation block of one token tile and one 128-chunk of the reduction axis: the
// tile's `rows` rows in the swizzled order the MMA reads, then the tile's scale-factor
// groups for the chunk's four 32-blocks, padded to a multiple of 1 KB.  One contiguous copy
// brings a block into shared memory.  A row holds the chunk's 128 activations:
//  - E4M3 (bf16 as two terms, or MXFP8): 128 bytes, 128-byte swizzle (16-byte unit u of
//    row n at unit u ^ (n % 8));
//  - E2M1 (MXFP4): 64 bytes of packed codes (element 2i in the low nibble of byte i),
//    64-byte swizzle (unit u of row n at unit u ^ ((n / 2) % 4)).
__host__ __device__ constexpr int packed_block_bytes(int rows, int row_bytes = kKChunk) {
  return (rows * row_bytes + sf_groups_of(rows) * kSfGroupBytes + 1023) / 1024 * 1024;
}
__host__ __device__ __forceinline__ int packed_unit_offset(int n, int u) { return n * kKChunk + ((u ^ (n & 7)) << 4); }
__host__ __device__ __forceinline__ int packed_unit_offset64(int n, int u) {
  return n * (kKChunk / 2) + ((u ^ ((n >> 1) & 3)) << 4);
}
__host__ __device__ __forceinline__ int packed_sf_offset(int rows, int n, int b, int row_bytes = kKChunk) {
  return rows * row_bytes + (n >> 7) * kSfGroupBytes + sf_byte_in_group(n & 127, b & 3);
}

// ---------------------------------------------------------------- MXFP4 (E2M1 + E8M0)
// The format of the pages (ewbang.com GPT-OSS article, section 量化: 4-bit values, one
// 8-bit scale per 32): block scale 2^s with s = floor(log2 amax) - 2 clamped to [-127, 127]
// (0 for an all-zero block), element = nearest E2M1 value of v / 2^s (ties to the even
// code), saturating at 6.  Used for the weights and, with MXFP4 activations, for the
// expert inputs and the SwiGLU outputs.

// E2M1 magnitude code (0..7) of a >= 0 (already divided by the block scale): the number of
// rounding thresholds between grid neighbours (0 .5 1 1.5 2 3 4 6) that a passes; ">" where
// a tie belongs to the lower (even) code, ">=" where it belongs to the upper one.
__device__ __forceinline__ int e2m1_code_of(float a) {
  int c = 0;
  c += a > 0.25f;   // tie -> 0
  c += a >= 0.75f;  // tie -> 1.0
  c += a > 1.25f;   // tie -> 1.0
  c += a >= 1.75f;  // tie -> 2.0
  c += a > 2.5f;    // tie -> 2.0
  c += a >= 3.5f;   // tie -> 4.0
  c += a > 5.0f;    // tie -> 4.0
  return c;
}

// ------------------------------------------------------------------ MXFP4 storage layout
// Weights [E][N][K] (moe_mxfp4.h) in tiles of 128 rows x 128 k: codes [E][NT][KC][128][64]
// (one contiguous 8 KB block per tile, row-major inside), scales [E][NT][KC][512] in the
// scale-factor layout above; NT = ceil(N/128), KC = ceil(K/128).  Gate_up tensors store
// rows in 128-row tiles of 64 gate rows + the 64 matching up rows.
constexpr int kCodeBlockBytes = 128 * kKChunk / 2;   // 8 KB

__host__ __device__ __forceinline__ int64_t mx_code_offset(int64_t e, int64_t row, int64_t k, int64_t N, int64_t K) {
  const int64_t nt = (N + 127) / 128, kc = kpad128(K) / kKChunk;
  return ((e * nt + row / 128) * kc + k / kKChunk) * kCodeBlockBytes + (row & 127) * (kKChunk / 2) +
         (k % kKChunk) / 2;
}
__host__ __device__ __forceinline__ int64_t gate_up_stored_row(int64_t n, int64_t I) {
  const int64_t part = n >= I ? 1 : 0, f = n - part * I;
  return (f / 64) * 128 + part * 64 + f % 64;
}

__host__ __device__ __forceinline__ int64_t mx_scale_offset(int64_t e, int64_t row, int64_t b, int64_t N, int64_t K) {
  const int64_t nt = (N + 127) / 128, kc = kpad128(K) / kKChunk;
  return ((e * nt + row / 128) * kc + b / 4) * kSfGroupBytes + sf_byte_in_group((int)(row & 127), (int)(b & 3));
}

// Carve-up of the caller's workspace (byte offsets, 256-byte aligned).
struct WsLayout {
  size_t status;    // int32 device status word (first device error wins)
  size_t counts;    // int32 [E] expert histogram, then int32 [4] (routing ticket), then int32
                    // [T * ceil(d/128)] combine arrivals; cleared at the start of every call
  size_t offsets;   // int32 [E+1]
  size_t ntiles;    // int32 [4]: number of token tiles
  size_t tile_base; // int32 [E]: first token tile of each expert
  size_t tiles;     // Tile [max_tiles]
  size_t topk_idx;  // int32 [T*k]
  size_t topk_w;    // f32 [T*k]
  size_t perm;      // int32 [P]   sorted position -> t*k + slot
  size_t inv;       // int32 [P]   t*k + slot -> sorted position
  size_t w_sorted;  // f32 [P]     routing weight of each sorted pair
  size_t xq;        // E4M3 [T][2][dp]   hi / lo terms of xe = bf16(RMSNorm(x)) (MXFP4: packed
                    // E2M1 codes in the first dp/2 bytes of each token's row)
  size_t xsf;       // E8M0 [T][2][dp/32] their scales
  size_t bpx;       // packed blocks [max_tiles][dp/128] of xe per token tile (gate_up's B)
  size_t bph;       // packed blocks [max_tiles][ip/128] of h per token tile (down's B)
  size_t ys;        // f32 [ksplit][P][d]  routing-weighted expert outputs (partial sums per
                    // reduction-axis split of the down GEMM), row t * k + slot of pair (t, slot)
  size_t total;
  int64_t max_tiles;
  int32_t tile_tokens;
  int32_t terms;     // rows per token fed to the MMAs: 2 (bf16 activations) or 1 (MXFP8, MXFP4)
  int32_t fp4;       // activations are MXFP4 (E2M1 rows of 64 bytes per chunk)
  int32_t ksplit;   // down GEMM reduction-axis splits (ys planes)
  int32_t dp, ip;   // d and I rounded up to 128
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline WsLayout ws_layout(const moe_dims& dm, int64_t T, int tile_tokens, int ksplit, int terms, int fp4) {
  WsLayout L{};
  const int64_t P = T * dm.top_k;
  const int row_bytes = fp4 ? kKChunk / 2 : kKChunk;
  L.tile_tokens = tile_tokens;
  L.ksplit = ksplit;
  L.terms = terms;
  L.fp4 = fp4;
  L.max_tiles = (P + tile_tokens - 1) / tile_tokens + dm.E;
  L.dp = (int32_t)kpad128(dm.d);
  L.ip = (int32_t)kpad128(dm.I);
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
  L.tile_base = take(4 * (size_t)dm.E);
  L.tiles = take(sizeof(Tile) * (size_t)L.max_tiles);
  L.topk_idx = take(4 * (size_t)P);
  L.topk_w = take(4 * (size_t)P);
  L.perm = take(4 * (size_t)P);
  L.inv = take(4 * (size_t)P);
  L.w_sorted = take(4 * (size_t)P);
  L.xq = take(2 * (size_t)T * L.dp);
  L.xsf = take(2 * (size_t)T * (L.dp / 32));
  L.bpx = take((size_t)L.max_tiles * (L.dp / kKChunk) * packed_block_bytes(terms * tile_tokens, row_bytes));
  L.bph = take((size_t)L.max_tiles * (L.ip / kKChunk) * packed_block_bytes(terms * tile_tokens, row_bytes));
  L.ys = take(4 * (size_t)ksplit * P * dm.d);
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
  int32_t* tile_base;
  Tile* tiles;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* perm;
  int32_t* inv;
  float* w_sorted;
  uint8_t* xq;
  uint8_t* xsf;
  uint8_t* bpx;
  uint8_t* bph;
  float* ys;
  uint8_t* bpx_end;    // ends of the buffers written at computed offsets (bounds checks)
  uint8_t* bph_end;
  float* ys_end;
  int64_t max_tiles;
  int32_t tile_tokens;
  int32_t terms;
  int32_t fp4;
  int32_t ksplit;
  int32_t dp, ip;
};

inline Ws ws_pointers(void* base, const WsLayout& L, int E) {
  char* b = static_cast<char*>(base);
  Ws w;
  w.status = reinterpret_cast<int32_t*>(b + L.status);
  w.counts = reinterpret_cast<int32_t*>(b + L.counts);
  w.offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  w.ntiles = reinterpret_cast<int32_t*>(b + L.ntiles);
  w.tile_base = reinterpret_cast<int32_t*>(b + L.tile_base);
  w.tiles = reinterpret_cast<Tile*>(b + L.tiles);
  w.topk_idx = reinterpret_cast<int32_t*>(b + L.topk_idx);
  w.topk_w = reinterpret_cast<float*>(b + L.topk_w);
  w.perm = reinterpret_cast<int32_t*>(b + L.perm);
  w.inv = reinterpret_cast<int32_t*>(b + L.inv);
  w.w_sorted = reinterpret_cast<float*>(b + L.w_sorted);
  w.xq = reinterpret_cast<uint8_t*>(b + L.xq);
  w.xsf = reinterpret_cast<uint8_t*>(b + L.xsf);
  w.bpx = reinterpret_cast<uint8_t*>(b + L.bpx);
  w.bph = reinterpret_cast<uint8_t*>(b + L.bph);
  w.ys = reinterpret_cast<float*>(b + L.ys);
  w.bpx_end = w.bph;
  w.bph_end = reinterpret_cast<uint8_t*>(b + L.ys);
  w.ys_end = reinterpret_cast<float*>(b + L.total);
  w.ticket = w.counts + E;
  w.arrivals = w.counts + E + 4;
  w.max_tiles = L.max_tiles;
  w.tile_tokens = L.tile_tokens;
  w.ksplit = L.ksplit;
  w.terms = L.terms;
  w.fp4 = L.fp4;
  w.dp = L.dp;
  w.ip = L.ip;
  return w;
}

// ------------------------------------------------------------ activations as E4M3 pairs
// The block-scaled MMA takes E4M3 activations with one E8M0 scale per 32 values.  A
// bf16 value v (8 significant bits) is carried as two terms: hi = RN_e4m3(v / 2^s1) and
// lo = RN_e4m3((v - hi * 2^s1) / 2^s2), where 2^s1 puts the block's largest |v| in
// [128, 256) and s2 = s1 - 4.  The residual is at most half a step of hi, i.e. at most
// 8 * 2^s1, so (v - hi * 2^s1) / 2^s2 <= 128 fits E4M3; it has at most 4 significant
// bits (bf16's 8 minus hi's 4), so lo is exact while it stays in E4M3's normal range.
// Hence hi * 2^s1 + lo * 2^s2 == v for every v of the block within a factor 2^13 of the
// largest, and within 2^-20 of the largest otherwise.

// fp32 -> bf16 bit pattern, round to nearest, ties to even.  A NaN stays a NaN (quiet,
// sign kept); the rounding carry alone could turn a NaN whose payload sits in the low 16
// bits into an infinity.
__device__ __forceinline__ uint16_t bf16_bits_rne(float f) {
  const uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// floor(log2(a)) for a finite a > 0 (normal or subnormal), exactly.
__device__ __forceinline__ int floor_log2f(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int e = (int)((bits >> 23) & 0xFF);
  if (e != 0) return e - 127;
  return (31 - __clz((int)(bits & 0x7FFFFF))) - 149;
}

// Scale exponent for a block whose largest magnitude is amax (0 for an all-zero block):
// amax / 2^s lands in [128, 256); s is clamped to [-122, 126] so that s - 4 stays a
// normal power of two (E8M0 bytes 1..253).
__device__ __forceinline__ int e4m3_block_exp(float amax) {
  if (!(amax > 0.f) || !(amax < INFINITY)) return 0;
  return max(-122, min(126, floor_log2f(amax) - 7));
}

__device__ __forceinline__ float pow2f(int s) { return __uint_as_float((uint32_t)(s + 127) << 23); }  // s in [-126, 127]

// Two fp32 values to E4M3 (round to nearest even, saturating); a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// E4M3 byte (low byte of q) back to fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t q) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(q & 0xFFu)));
  return __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFFu)));
}

// Warp-cooperative split of 32-value blocks: each lane holds V consecutive values of a
// block spread over 32/V consecutive lanes (V = 1: one block per warp; V = 2: two).
// Returns this lane's hi / lo bytes (value i in byte i) and the block's two scale bytes.
template <int V>
__device__ __forceinline__ void e4m3_split(const float (&v)[V], uint32_t& hi, uint32_t& lo, uint32_t& sf_hi,
                                           uint32_t& sf_lo) {
  constexpr int kLanes = 32 / V;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = kLanes / 2; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int s1 = e4m3_block_exp(amax), s2 = s1 - 4;
  const float inv1 = pow2f(-s1), sc1 = pow2f(s1), inv2 = pow2f(-s2);
  hi = 0u;
  lo = 0u;
  if constexpr (V % 2 == 0) {
    // two values per conversion (each rounded on its own, as below)
#pragma unroll
    for (int i = 0; i < V; i += 2) {
      const uint32_t q2 = e4m3x2(v[i] * inv1, v[i + 1] * inv1);
      hi |= q2 << (8 * i);
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)q2));
      const float d0 = __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFFu)));
      const float d1 = __half2float(__ushort_as_half((uint16_t)(h2 >> 16)));
      const float r0 = v[i] - d0 * sc1, r1 = v[i + 1] - d1 * sc1;   // exact
      lo |= e4m3x2(r0 * inv2, r1 * inv2) << (8 * i);
    }
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const uint32_t q = e4m3x2(v[i] * inv1, 0.f) & 0xFFu;
      hi |= q << (8 * i);
      const float r = v[i] - e4m3_to_f32(q) * sc1;   // exact
      lo |= (e4m3x2(r * inv2, 0.f) & 0xFFu) << (8 * i);
    }
  }
  sf_hi = (uint32_t)(s1 + 127);
  sf_lo = (uint32_t)(s2 + 127);
}

// Warp-cooperative MXFP4 quantization of 32-value blocks, in the lane layout of e4m3_split
// (each lane holds V consecutive values of a block spread over 32/V lanes), by the rule of
// the weights (see e2m1_code_of).  Returns this lane's E2M1 codes (value i in bits 4i..4i+3;
// bit 3 of a code is the sign, set only on non-zero codes) and the block's scale byte.
template <int V>
__device__ __forceinline__ void e2m1_quant(const float (&v)[V], uint32_t& codes, uint32_t& sf) {
  constexpr int kLanes = 32 / V;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = kLanes / 2; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int s = 0;
  if (amax > 0.f && amax < INFINITY) s = max(-127, min(127, floor_log2f(amax) - 2));
  codes = 0u;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    int c = e2m1_code_of(ldexpf(fabsf(v[i]), -s));   // exact power-of-two scaling
    if (v[i] < 0.f && c != 0) c |= 8;
    codes |= (uint32_t)c << (4 * i);
  }
  sf = (uint32_t)(s + 127);
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
  // Optional outputs in place of (or beside) y:
  float* y_partial;          // [T][d] fp32 sum_j w_j o_j without the residual (a slice of I)
  const float* next_norm_w;  // [d]: also write y_norm = bf16(RMSNorm(y) * next_norm_w)
  float next_eps;
  uint16_t* y_norm;          // [T][d] bf16
  Ws ws;
  cudaStream_t stream;
  EventRec* ev;
  int32_t inject_timeout;  // test hook: withhold one pipeline arrival in the gate_up kernel
  int32_t fuse_group;      // small batches: the routing kernel also groups (and packs the tiles)
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

// As launch_kernel, in clusters of `cluster_x` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                                  unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
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

// Record the first device-side error in the status word.
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Stores at computed offsets (packed blocks, expert outputs, outputs, quantized weights) go
// through in_bounds(p, lo, hi, status): with MOE_DEBUG_BOUNDS defined (the bounds-checking
// build) a store outside [lo, hi) is skipped and MOE_ERR_BOUNDS recorded; otherwise the
// check compiles away.
template <class T, class U>
__device__ __forceinline__ bool in_bounds(const T* p, const U* lo, const U* hi, int32_t* status) {
#ifdef MOE_DEBUG_BOUNDS
  const char* c = reinterpret_cast<const char*>(p);
  if (c >= reinterpret_cast<const char*>(lo) && c + sizeof(T) <= reinterpret_cast<const char*>(hi)) return true;
  set_status(status, MOE_ERR_BOUNDS);
  return false;
#else
  (void)p; (void)lo; (void)hi; (void)status;
  return true;
#endif
}

// ----------------------------------------------------------------------------------
// Top-k (value desc, index asc) + softmax over the selected logits for one token, by one
// warp; the lane holding logit e is lane e % 32.  Writes the outputs and the histogram.
// ----------------------------------------------------------------------------------
template <int NJ>
__device__ __forceinline__ void warp_topk_softmax(float (&l)[NJ], int E, int k, int64_t t, const FwdArgs& a) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    if (lane + 32 * j < E && !isfinite(l[j])) {
      bad = true;
      l[j] = -INFINITY;
    }
    if (lane + 32 * j >= E) l[j] = -INFINITY;
  }
  if (__any_sync(0xffffffffu, bad)) set_status(a.ws.status, MOE_ERR_NONFINITE);
  float lsel = 0.f, lmax = 0.f, z = 0.f;
  int esel = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
      const int e = lane + 32 * jj;
      if (e < E && (l[jj] > bv || (l[jj] == bv && e < be))) {
        bv = l[jj];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be >= E) be = j;  // only when every logit was non-finite; the status already says so
    if (j == 0) lmax = bv;
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj)
      if (lane + 32 * jj == be) l[jj] = -INFINITY;
    const float ex = expf(bv - lmax);
    z += ex;
    if (lane == j) {
      lsel = ex;
      esel = be;
    }
  }
  if (lane < k) {
    a.ws.topk_idx[t * k + lane] = esel;
    a.ws.topk_w[t * k + lane] = lsel / z;
    atomicAdd(&a.ws.counts[esel], 1);
  }
}

// --------------------------------------------------------------------------- launchers
// Each returns the number of kernels it launched (>= 0) or -1 on a launch error.
int launch_quantize(const float* w, int32_t E, int32_t N, int32_t K, int32_t role, uint8_t* codes,
                    uint8_t* scales, int32_t* status, cudaStream_t st);
int launch_route(const FwdArgs& a);     // norm + router + top-k + E4M3 split, grouping, packing
int launch_route_mma(const FwdArgs& a); // the same first step for large batches, logits on the tensor cores
bool route_mma_fits(int E, int d);      // its shared memory fits
int launch_combine(const FwdArgs& a);   // y = x + sum_j ys[inv] (or the partial sum, or y and y_norm)
// y = bf16(x + s) for a dense fp32 s [T][d], and optionally y_norm (one pass per row)
int launch_residual_norm(int32_t T, int32_t d, const uint16_t* x, const float* s, const float* norm_w, float eps,
                         uint16_t* y, uint16_t* y_norm, cudaStream_t st);
int launch_experts(const FwdArgs& a);   // block-scaled tcgen05 expert MLPs (gate_up, down)
int expert_tile_tokens(int path, int terms);   // token tile of a path
int expert_down_split(int path);        // reduction-axis splits of a path's down GEMM
moe_status validate_dims(const moe_dims* dims, int32_t T);   // the argument checks of every call

}  // namespace moe
