// MXFP4 quantization, RMSNorm + router + top-k, grouping, tile packing and combine.
//
// Layer definition (web pages on gpt-oss):
//  - RMSNorm: "From GPT-2 to gpt-oss" (新智元 translation), sec. 7: divide by the
//    RMS, no mean subtraction, no bias; rms_norm_eps 1e-5 (llm-atlas GPT-OSS 20B
//    config table).
//  - Router + top-k: ewbang.com GPT-OSS article, section 混合专家模型: a small
//    network scores the experts, several are chosen per token and weighted
//    (e.g. 0.7 x NN2 + 0.3 x NN4); top-4 of 32 / 128.
//  - MXFP4: same article, section 量化: 4-bit values, one 8-bit scale per 32
//    parameters, 4.25 bits per parameter.
#include <cuda_fp16.h>
#include <algorithm>
#include <atomic>
#include <cfloat>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }


// ----------------------------------------------------------------------------------
// Quantization: one warp per 32-value block, lane i holds element i.
// Scale exponent s = floor(log2 amax) - 2 from the exponent bits of amax (exact);
// the E2M1 code of |x| * 2^-s is the number of rounding thresholds it passes,
// each threshold taking ties toward the even code.
// ----------------------------------------------------------------------------------
__global__ void quantize_kernel(const float* __restrict__ w, int64_t nblocks, int32_t N, int32_t K, int32_t role,
                                uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int32_t* status,
                                const uint8_t* codes_end, const uint8_t* scales_end) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int kb_per_row = K / 32;
  for (int64_t b = warp; b < nblocks; b += nwarps) {
    const int64_t row = b / kb_per_row;          // row of [E*N]
    const int kb = (int)(b - row * kb_per_row);
    const float v = w[b * 32 + lane];
    const float a = fabsf(v);
    const bool finite = isfinite(v);
    float amax = a;
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const bool all_finite = __all_sync(0xffffffffu, finite);
    int s = 0;
    if (amax > 0.f && all_finite) {
      const uint32_t bits = __float_as_uint(amax);
      int e = (int)((bits >> 23) & 0xFF);
      int fl;
      if (e != 0) fl = e - 127;                                  // normal: floor(log2) = exponent
      else fl = (31 - __clz((int)(bits & 0x7FFFFF))) - 149;      // subnormal: m * 2^-149
      s = max(-127, min(127, fl - 2));
    }
    // x * 2^-s exactly (power-of-two scaling; ldexpf is exact when no under/overflow
    // changes a value that matters: scaled values below 0.25 all round to code 0).
    const float scaled = ldexpf(a, -s);
    int c = all_finite ? e2m1_code_of(scaled) : 0;
    if (v < 0.f && c != 0) c |= 8;
    const int hi = __shfl_down_sync(0xffffffffu, c, 1);
    const int64_t e_idx = row / N;
    const int64_t n = row - e_idx * N;
    const int64_t srow = role == MOE_WEIGHT_GATE_UP ? gate_up_stored_row(n, N / 2) : n;
    uint8_t* qc = codes + mx_code_offset(e_idx, srow, 32 * kb + lane, N, K);
    if ((lane & 1) == 0 && in_bounds(qc, codes, codes_end, status)) *qc = (uint8_t)(c | (hi << 4));
    if (lane == 0) {
      uint8_t* qs = scales + mx_scale_offset(e_idx, srow, kb, N, K);
      if (in_bounds(qs, scales, scales_end, status)) *qs = all_finite ? (uint8_t)(s + 127) : (uint8_t)0xFF;
      if (!all_finite) set_status(status, MOE_ERR_NONFINITE);
    }
  }
}

// ----------------------------------------------------------------------------------
// Grouping for a small batch, run by the routing CTA that finished last
// (all others have published their top-k, counts and xq rows before taking a ticket).
// Pairs are listed per expert in token order: one warp walks the tokens in order and
// hands each of a token's k (distinct) experts the next free position of that expert.
// Deterministic: positions depend on counts and token order only.
// ----------------------------------------------------------------------------------
// Chunk c of token t's E4M3 rows (hi, lo) and their scales into the packed block of
// token tile `tile`, MMA columns 2*col (hi) and 2*col + 1 (lo).  One warp: lanes 0-15
// move the 16 16-byte units, lanes 16-23 the eight scale bytes.
template <bool FP4>
__device__ __forceinline__ void pack_pair_chunk(const FwdArgs& a, int t, int tile, int col, int c) {
  const int lane = threadIdx.x & 31;
  const int dp = a.ws.dp, nb = a.d / 32, bt = a.ws.tile_tokens, kc = dp / kKChunk, terms = a.ws.terms;
  const int rows = terms * bt;
  if (FP4) {   // MXFP4: one 64-byte row of packed codes; lanes 0-3 move it, 16-19 the scales
    uint8_t* block = a.ws.bpx + ((int64_t)tile * kc + c) * packed_block_bytes(rows, kKChunk / 2);
    if (lane < 4) {
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(a.ws.xq + (int64_t)t * 2 * dp + c * (kKChunk / 2)) + lane);
      uint4* q = reinterpret_cast<uint4*>(block + packed_unit_offset64(col, lane));
      if (in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status)) *q = v;
    } else if (lane >= 16 && lane < 20) {
      const int b = 4 * c + (lane - 16);
      uint8_t* q = block + packed_sf_offset(rows, col, b, kKChunk / 2);
      if (b < nb && in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status))
        *q = __ldcg(a.ws.xsf + (int64_t)t * 2 * (dp / 32) + b);
    }
    return;
  }
  uint8_t* block = a.ws.bpx + ((int64_t)tile * kc + c) * packed_block_bytes(rows);
  if (lane < 16) {   // (units past d are never read by the MMAs)
    const int term = lane >> 3, u = lane & 7;
    if (term < terms) {
      const uint4 v =
          __ldcg(reinterpret_cast<const uint4*>(a.ws.xq + (int64_t)t * 2 * dp + term * dp + c * kKChunk) + u);
      uint4* q = reinterpret_cast<uint4*>(block + packed_unit_offset(terms * col + term, u));
      if (in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status)) *q = v;
    }
  } else if (lane < 24) {
    const int term = (lane - 16) >> 2, b = 4 * c + ((lane - 16) & 3);
    uint8_t* q = block + packed_sf_offset(rows, terms * col + term, b);
    if (term < terms && b < nb && in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status))
      *q = __ldcg(a.ws.xsf + (int64_t)t * 2 * (dp / 32) + term * (dp / 32) + b);
  }
}

__device__ void group_block(const FwdArgs& a, int tile_tokens) {
  __shared__ int s_off[257];
  __shared__ int s_cur[256];
  __shared__ int s_tb[257];
  __shared__ int s_perm_tok[kFusedGroupMaxT * 32];
  __shared__ int s_perm_e[kFusedGroupMaxT * 32];
  const int E = a.E, k = a.k, T = a.T, P = T * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp == 0) {
    // exclusive scans of counts and of tiles-per-expert over E <= 256 (8 experts per lane)
    int c[8], nt[8], sc = 0, st = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      c[j] = (e < E) ? __ldcg(a.ws.counts + e) : 0;
      nt[j] = (c[j] + tile_tokens - 1) / tile_tokens;
      sc += c[j];
      st += nt[j];
    }
    int ic = sc, it = st;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yc = __shfl_up_sync(0xffffffffu, ic, o), yt = __shfl_up_sync(0xffffffffu, it, o);
      if (lane >= o) {
        ic += yc;
        it += yt;
      }
    }
    int oc = ic - sc, ot = it - st;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E) {
        s_off[e] = oc;
        s_tb[e] = ot;
        s_cur[e] = 0;
        a.ws.offsets[e] = oc;
        a.ws.tile_base[e] = ot;
      }
      oc += c[j];
      ot += nt[j];
    }
    if (lane == 31) {
      a.ws.offsets[E] = oc;
      a.ws.ntiles[0] = ot;
    }
  }
  __syncthreads();
  // token tiles of every expert
  for (int e = warp; e < E; e += (int)(blockDim.x >> 5)) {
    const int base = s_tb[e];
    const int c_e = (e + 1 < E ? s_off[e + 1] : P) - s_off[e];
    for (int i = lane; i * tile_tokens < c_e; i += 32) {
      Tile tl;
      tl.e = e;
      tl.row0 = s_off[e] + i * tile_tokens;
      tl.rows = min(tile_tokens, c_e - i * tile_tokens);
      tl.pad = 0;
      a.ws.tiles[base + i] = tl;
    }
  }
  // every pair's expert id, loaded once (staged in s_perm_tok until the walk is done)
  for (int q = tid; q < P; q += blockDim.x) s_perm_tok[q] = __ldcg(a.ws.topk_idx + q);
  __syncthreads();
  if (warp == 0) {
    for (int t = 0; t < T; ++t) {
      if (lane < k) {
        const int q = t * k + lane;
        const int e = s_perm_tok[q];
        const int pos = s_off[e] + s_cur[e]++;   // a token's k experts are distinct
        s_perm_e[pos] = e | (q << 9);            // (E <= 256, q < 64 * 32)
      }
      __syncwarp();
    }
  }
  __syncthreads();
  for (int pos = tid; pos < P; pos += blockDim.x) {
    const int v = s_perm_e[pos], q = v >> 9;
    a.ws.perm[pos] = q;
    a.ws.inv[q] = pos;
    a.ws.w_sorted[pos] = __ldcg(a.ws.topk_w + q);
  }
}

// ----------------------------------------------------------------------------------
// Small batches: one cluster of kTokCluster CTAs (256 threads each) per token.  Every CTA
// of the cluster normalizes the token's row into shared memory (fp32; the row is small,
// each CTA reads it), writes the activation format of its share of the 32-blocks, and
// computes the logits of its share of the experts (warp w: experts first + w, + 8, ...,
// each lane issuing all of its 16-byte loads of the router row before the FMAs); the
// logits go into the shared memory of the cluster's first CTA, which after the cluster
// barrier selects the top-k.  Spreading a token's experts over the cluster spreads the
// router rows' bytes over four SMs.
// ----------------------------------------------------------------------------------
constexpr int kTokCluster = 4;
constexpr int kTokThreads = 256;
constexpr int kTokWarps = kTokThreads / 32;
constexpr int kTokBatch = 12;   // router-row loads in flight per lane

template <int NJ>
__global__ void __launch_bounds__(kTokThreads) route_token_kernel(FwdArgs a) {
  extern __shared__ float smem[];
  pdl_trigger();
  const int d = a.d, E = a.E;
  float* s_xn = smem;          // [d]
  float* s_l = smem + d;       // [32*NJ] logits (in the cluster's first CTA)
  __shared__ float s_red[kTokWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)ptx::cluster_ctarank();
  const int64_t t = blockIdx.x / kTokCluster;
  const uint16_t* xr = a.x + t * d;
  float ss = 0.f;
  for (int i = tid * 8; i < d; i += kTokThreads * 8) {
    const uint4 q = *reinterpret_cast<const uint4*>(xr + i);
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(wv[j] << 16), hi = __uint_as_float(wv[j] & 0xFFFF0000u);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
      s_xn[i + 2 * j] = lo;
      s_xn[i + 2 * j + 1] = hi;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) s_red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kTokWarps; ++w) tot += s_red[w];
  const float r = 1.0f / sqrtf(tot / (float)d + a.eps);
  for (int i = tid * 2; i < d; i += 2 * kTokThreads) {
    s_xn[i] = s_xn[i] * r * a.norm_w[i];
    s_xn[i + 1] = s_xn[i + 1] * r * a.norm_w[i + 1];
  }
  __syncthreads();
  {
    // xe = bf16(xn) as E4M3 hi / lo terms (or one MXFP8 term, or MXFP4 codes): this CTA's
    // 32-blocks, one per warp at a time
    const int dp = a.ws.dp, nb = d / 32;
    uint8_t* xq = a.ws.xq + t * 2 * dp;
    uint8_t* sf = a.ws.xsf + t * 2 * (dp / 32);
    for (int b = rank * nb / kTokCluster + warp; b < (rank + 1) * nb / kTokCluster; b += kTokWarps) {
      const float v[1] = {bf16_to_f32(bf16_bits_rne(s_xn[32 * b + lane]))};
      if (a.ws.fp4) {   // MXFP4 activations: packed E2M1 codes, two per byte
        uint32_t c, s1;
        e2m1_quant<1>(v, c, s1);
        const uint32_t c_hi = __shfl_down_sync(0xffffffffu, c, 1);
        if ((lane & 1) == 0) xq[16 * b + lane / 2] = (uint8_t)(c | (c_hi << 4));
        if (lane == 0) sf[b] = (uint8_t)s1;
        continue;
      }
      uint32_t hi, lo, s1, s2;
      e4m3_split<1>(v, hi, lo, s1, s2);
      xq[32 * b + lane] = (uint8_t)hi;
      xq[dp + 32 * b + lane] = (uint8_t)lo;
      if (lane == 0) {
        sf[b] = (uint8_t)s1;
        sf[dp / 32 + b] = (uint8_t)s2;
      }
    }
  }
  const int n4 = d / 4;
  for (int e = rank * E / kTokCluster + warp; e < (rank + 1) * E / kTokCluster; e += kTokWarps) {
    const float4* wr = reinterpret_cast<const float4*>(a.router_w + (int64_t)e * d);
    float acc = 0.f;
    // batches of kTokBatch 16-byte loads per lane, all issued before their FMAs
    for (int base = 0; base < n4; base += 32 * kTokBatch) {
      float4 w4[kTokBatch];
#pragma unroll
      for (int j = 0; j < kTokBatch; ++j) {
        const int i4 = base + lane + 32 * j;
        w4[j] = (i4 < n4) ? wr[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < kTokBatch; ++j) {
        const int i4 = base + lane + 32 * j;
        if (i4 < n4) {
          const float4 x4 = reinterpret_cast<const float4*>(s_xn)[i4];
          acc = fmaf(w4[j].x, x4.x, acc);
          acc = fmaf(w4[j].y, x4.y, acc);
          acc = fmaf(w4[j].z, x4.z, acc);
          acc = fmaf(w4[j].w, x4.w, acc);
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) ptx::st_cluster_f32(ptx::mapa_shared(&s_l[e], 0), acc + (a.router_b ? a.router_b[e] : 0.f));
  }
  ptx::cluster_sync();   // every logit of the token is in the first CTA's shared memory
  if (rank != 0) return;
  if (warp == 0) {
    float l[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) l[j] = (lane + 32 * j < E) ? s_l[lane + 32 * j] : -INFINITY;
    warp_topk_softmax<NJ>(l, E, a.k, t, a);
  }
  if (a.fuse_group) {
    // Publish this token (top-k, counts, xq rows: the other CTAs of the cluster wrote
    // theirs before the cluster barrier), then take a ticket; the last token's CTA groups.
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(a.ws.ticket, 1) == a.T - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      group_block(a, a.fuse_group);
    }
  }
}

// ----------------------------------------------------------------------------------
// Large batches: fused RMSNorm + router + top-k + softmax, kRT tokens per CTA, 256
// threads.  The reduction axis is walked in chunks of RK through a ring of NS cp.async
// stages, each holding the chunk's bf16 x rows of the CTA's tokens and the router rows
// [E][RK] (fp32, rows padded by 4 floats so that the float4 reads of 32 consecutive
// experts hit distinct banks).  Per chunk, warp w first normalizes tokens 2w and 2w + 1
// (xn = x / rms * gamma, fp32) and stores their E4M3 hi / lo terms and scales; then warp
// w takes the chunk's columns [RK/8 w, RK/8 (w + 1)): each lane keeps those router
// values of its experts (lane + 32 j) in registers and accumulates them against every
// token's xn (broadcast reads).  The eight warps' partial logits are added at the end
// in warp order.  Outputs: xq / xsf, topk_idx, topk_w, expert histogram.
// ----------------------------------------------------------------------------------
constexpr int kRT = 16;                  // tokens per CTA
constexpr int kTokenKernelMaxT = 256;    // up to this many tokens: one CTA per token
#ifndef MOE_ROUTE_MMA_MIN_CTAS
#define MOE_ROUTE_MMA_MIN_CTAS 64
#endif
constexpr int kRouteMmaMinCtas = MOE_ROUTE_MMA_MIN_CTAS;   // the tensor-core router from this many 128-token CTAs

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int NJ, int RK, int NS>
struct RouteTilesCfg {
  static constexpr int EP = 32 * NJ;
  static constexpr int WST = RK + 4;                       // router row stride (floats)
  static constexpr int W_FLOATS = EP * WST;                // one stage of router rows
  static constexpr int X_HALVES = kRT * RK;                // one stage of x (bf16)
  static constexpr int KW = RK / 8;                        // columns of a chunk per warp
  static constexpr size_t STAGES = sizeof(float) * (NS * W_FLOATS + kRT * RK) + 2 * NS * X_HALVES;
  // RMSNorm weights (d floats) follow the stages / partials
  static constexpr size_t PARTIALS = sizeof(float) * 8 * kRT * EP;   // final reduction (reuses the stages)
  static constexpr size_t MAIN = STAGES > PARTIALS ? STAGES : PARTIALS;
  static size_t smem(int d) { return MAIN + sizeof(float) * (size_t)d; }
  static_assert(KW % 4 == 0, "float4 columns per warp");
};

template <int NJ, int RK, int NS, bool FP4>
__global__ void __launch_bounds__(256) route_tiles_kernel(FwdArgs a) {
  using C = RouteTilesCfg<NJ, RK, NS>;
  extern __shared__ __align__(16) float smem[];
  float* s_w = smem;                                        // [NS][EP][WST]
  float* s_xn = smem + NS * C::W_FLOATS;                   // [kRT][RK]
  uint16_t* s_x = reinterpret_cast<uint16_t*>(s_xn + kRT * RK);  // [NS][kRT][RK]
  float* s_g = smem + C::MAIN / sizeof(float);             // [d] RMSNorm weights
  __shared__ float s_r[kRT];
  pdl_trigger();
  const int E = a.E, d = a.d, k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRT;
  const int nt = min(kRT, a.T - t0);
  const int nchunks = d / RK;
  const int dp = a.ws.dp;

  auto issue = [&](int c) {   // chunk c into stage c % NS
    const int st = c % NS, k0 = c * RK;
    for (int i = tid; i < kRT * (RK / 8); i += 256) {   // x: 16-byte pieces
      const int tt = i / (RK / 8), q = i - tt * (RK / 8);
      if (tt < nt) cp_async16(s_x + (st * kRT + tt) * RK + q * 8, a.x + (int64_t)(t0 + tt) * d + k0 + q * 8);
    }
    for (int i = tid; i < E * (RK / 4); i += 256) {     // router rows: 16-byte pieces
      const int e = i / (RK / 4), q = i - e * (RK / 4);
      cp_async16(s_w + (st * C::EP + e) * C::WST + q * 4, a.router_w + (int64_t)e * d + k0 + q * 4);
    }
  };
  for (int c = 0; c < NS - 1; ++c) {
    if (c < nchunks) issue(c);
    cp_async_commit();
  }

  for (int i = tid * 4; i < d; i += 256 * 4) *reinterpret_cast<float4*>(s_g + i) = *reinterpret_cast<const float4*>(a.norm_w + i);
  // 1 / rms of the warp's two tokens (overlaps the first chunks' copies)
  for (int h = 0; h < 2; ++h) {
    const int tt = 2 * warp + h;
    float ss = 0.f;
    if (tt < nt) {
      const uint16_t* xr = a.x + (int64_t)(t0 + tt) * d;
      for (int i = lane * 8; i < d; i += 256) {
        const uint4 q = *reinterpret_cast<const uint4*>(xr + i);
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = __uint_as_float(wv[j] << 16), hi = __uint_as_float(wv[j] & 0xFFFF0000u);
          ss = fmaf(lo, lo, ss);
          ss = fmaf(hi, hi, ss);
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_r[tt] = 1.0f / sqrtf(ss / (float)d + a.eps);
  }
  __syncwarp();

  float acc[kRT][NJ];   // partial logits of this warp's columns, all tokens
#pragma unroll
  for (int t = 0; t < kRT; ++t)
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[t][j] = 0.f;

  for (int c = 0; c < nchunks; ++c) {
    if (c + NS - 1 < nchunks) issue(c + NS - 1);
    cp_async_commit();
    cp_async_wait<NS - 1>();
    __syncthreads();
    const int st = c % NS, k0 = c * RK;
    // normalize this warp's tokens, split into E4M3 terms (warp-private rows of s_xn)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int tt = 2 * warp + h;
      if (tt < nt) {   // uniform per warp
        const float r = s_r[tt];
        uint8_t* xq = a.ws.xq + (int64_t)(t0 + tt) * 2 * dp;
        uint8_t* sf = a.ws.xsf + (int64_t)(t0 + tt) * 2 * (dp / 32);
        if (RK == 64) {
          const int kk = 2 * lane;
          const uint32_t pr = *reinterpret_cast<const uint32_t*>(s_x + (st * kRT + tt) * RK + kk);
          const float v0 = __uint_as_float(pr << 16) * r * s_g[k0 + kk];
          const float v1 = __uint_as_float(pr & 0xFFFF0000u) * r * s_g[k0 + kk + 1];
          s_xn[tt * RK + kk] = v0;
          s_xn[tt * RK + kk + 1] = v1;
          const float v[2] = {bf16_to_f32(bf16_bits_rne(v0)), bf16_to_f32(bf16_bits_rne(v1))};
          if (FP4) {   // MXFP4 activations: this lane's two codes are one byte
            uint32_t c, s1;
            e2m1_quant<2>(v, c, s1);
            xq[(k0 + kk) / 2] = (uint8_t)c;
            if ((lane & 15) == 0) sf[(k0 + kk) / 32] = (uint8_t)s1;
            continue;
          }
          uint32_t hi, lo, s1, s2;
          e4m3_split<2>(v, hi, lo, s1, s2);   // lanes 0-15: block k0/32, 16-31: the next
          *reinterpret_cast<uint16_t*>(xq + k0 + kk) = (uint16_t)hi;
          *reinterpret_cast<uint16_t*>(xq + dp + k0 + kk) = (uint16_t)lo;
          if ((lane & 15) == 0) {
            sf[(k0 + kk) / 32] = (uint8_t)s1;
            sf[dp / 32 + (k0 + kk) / 32] = (uint8_t)s2;
          }
        } else {   // RK == 32: one 32-block per chunk, one value per lane
          const float v0 = bf16_to_f32(s_x[(st * kRT + tt) * RK + lane]) * r * s_g[k0 + lane];
          s_xn[tt * RK + lane] = v0;
          const float v[1] = {bf16_to_f32(bf16_bits_rne(v0))};
          if (FP4) {
            uint32_t c, s1;
            e2m1_quant<1>(v, c, s1);
            const uint32_t c_hi = __shfl_down_sync(0xffffffffu, c, 1);
            if ((lane & 1) == 0) xq[(k0 + lane) / 2] = (uint8_t)(c | (c_hi << 4));
            if (lane == 0) sf[k0 / 32] = (uint8_t)s1;
            continue;
          }
          uint32_t hi, lo, s1, s2;
          e4m3_split<1>(v, hi, lo, s1, s2);
          xq[k0 + lane] = (uint8_t)hi;
          xq[dp + k0 + lane] = (uint8_t)lo;
          if (lane == 0) {
            sf[k0 / 32] = (uint8_t)s1;
            sf[dp / 32 + k0 / 32] = (uint8_t)s2;
          }
        }
      }
    }
    __syncthreads();   // every warp's xn rows of this chunk are in place
    // acc[t][j] += router_w[lane + 32 j][columns of warp w] . xn[t][same columns]
    const float* wst = s_w + st * C::W_FLOATS;
    const int kw = warp * C::KW;
#pragma unroll
    for (int q = 0; q < C::KW; q += 4) {
      float4 w4[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) w4[j] = *reinterpret_cast<const float4*>(wst + (lane + 32 * j) * C::WST + kw + q);
#pragma unroll
      for (int t = 0; t < kRT; ++t) {
        const float4 xv = *reinterpret_cast<const float4*>(s_xn + t * RK + kw + q);
#pragma unroll
        for (int j = 0; j < NJ; ++j)
          acc[t][j] = fmaf(w4[j].x, xv.x, fmaf(w4[j].y, xv.y, fmaf(w4[j].z, xv.z, fmaf(w4[j].w, xv.w, acc[t][j]))));
      }
    }
    __syncthreads();   // stage st and the xn rows are refilled by the next iteration
  }
  cp_async_wait<0>();

  // add the warps' partial logits in warp order (router stages reused: [8][kRT][EP])
  float* s_part = s_w;
#pragma unroll
  for (int t = 0; t < kRT; ++t)
#pragma unroll
    for (int j = 0; j < NJ; ++j) s_part[(warp * kRT + t) * C::EP + lane + 32 * j] = acc[t][j];
  __syncthreads();
  // top-k + softmax: warp w takes tokens 2w and 2w + 1 (lane holds experts lane + 32 j)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int tt = 2 * warp + h;
    if (tt < nt) {
      float l[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += s_part[(w * kRT + tt) * C::EP + e];
        l[j] = (e < E) ? v + (a.router_b ? a.router_b[e] : 0.f) : -INFINITY;
      }
      warp_topk_softmax<NJ>(l, E, k, t0 + tt, a);
    }
  }
}

// ----------------------------------------------------------------------------------
// Grouping: CTA e lists expert e's pairs in token order (exclusive block scan of the
// per-token match flags), writes perm / inv / w_sorted, its offsets entry and its
// token tiles.  Deterministic: every position is a count, no order of atomics.
// ----------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) group_kernel(FwdArgs a, int tile_tokens) {
  __shared__ int s_warp[32];
  __shared__ int s_base, s_tile_base, s_total_tiles, s_off;
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.x, E = a.E, k = a.k, T = a.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    int off = 0, tb = 0, tot = 0;
    for (int q = 0; q < E; ++q) {
      const int c = a.ws.counts[q];
      const int nt = (c + tile_tokens - 1) / tile_tokens;
      if (q < e) {
        off += c;
        tb += nt;
      }
      tot += nt;
    }
    s_off = off;
    s_tile_base = tb;
    s_total_tiles = tot;
    s_base = 0;
  }
  __syncthreads();
  const int off = s_off;
  const int cnt = a.ws.counts[e];
  a.ws.offsets[e] = off;
  if (e == E - 1) a.ws.offsets[E] = off + cnt;
  if (e == 0) a.ws.ntiles[0] = s_total_tiles;
  if (tid == 0) a.ws.tile_base[e] = s_tile_base;
  for (int i = tid; i * tile_tokens < cnt; i += blockDim.x) {
    Tile tl;
    tl.e = e;
    tl.row0 = off + i * tile_tokens;
    tl.rows = min(tile_tokens, cnt - i * tile_tokens);
    tl.pad = 0;
    a.ws.tiles[s_tile_base + i] = tl;
  }
  for (int t0 = 0; t0 < T; t0 += blockDim.x) {
    const int t = t0 + tid;
    int slot = -1;
    if (t < T)
      for (int s = 0; s < k; ++s)
        if (a.ws.topk_idx[(int64_t)t * k + s] == e) slot = s;
    const unsigned m = __ballot_sync(0xffffffffu, slot >= 0);
    if (lane == 0) s_warp[warp] = __popc(m);
    __syncthreads();
    if (warp == 0) {
      int v = (lane < (int)(blockDim.x >> 5)) ? s_warp[lane] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      s_warp[lane] = incl - v;  // exclusive prefix of the warps
    }
    __syncthreads();
    if (slot >= 0) {
      const int pos = off + s_base + s_warp[warp] + __popc(m & ((1u << lane) - 1u));
      const int q = t * k + slot;
      a.ws.perm[pos] = q;
      a.ws.inv[q] = pos;
      a.ws.w_sorted[pos] = a.ws.topk_w[q];
    }
    __syncthreads();
    if (tid == blockDim.x - 1) s_base += s_warp[warp] + __popc(m);
    __syncthreads();
  }
}

// All chunks of token t's rows and scales into token tile `tile`'s packed blocks.  One
// warp; each lane keeps four 16-byte copies in flight.
template <bool FP4>
__device__ __forceinline__ void pack_pair(const FwdArgs& a, int t, int tile, int col) {
  const int lane = threadIdx.x & 31;
  const int dp = a.ws.dp, nb = a.d / 32, bt = a.ws.tile_tokens, kc = dp / kKChunk, terms = a.ws.terms;
  const int rows_t = terms * bt;
  if (FP4) {   // MXFP4: per chunk one 64-byte row of packed codes (4 units) and 4 scales
    const int bb = packed_block_bytes(rows_t, kKChunk / 2);
    uint8_t* blocks = a.ws.bpx + (int64_t)tile * kc * bb;
    const uint8_t* row = a.ws.xq + (int64_t)t * 2 * dp;
    for (int i = lane; i < kc * 4; i += 32) {
      const int c = i >> 2, u = i & 3;
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(row + c * (kKChunk / 2)) + u);
      uint4* q = reinterpret_cast<uint4*>(blocks + (int64_t)c * bb + packed_unit_offset64(col, u));
      if (in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status)) *q = v;
    }
    const uint8_t* sf = a.ws.xsf + (int64_t)t * 2 * (dp / 32);
    for (int b = lane; b < nb; b += 32) {
      uint8_t* q = blocks + (int64_t)(b / 4) * bb + packed_sf_offset(rows_t, col, b, kKChunk / 2);
      if (in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status)) *q = __ldcg(sf + b);
    }
    return;
  }
  const int bb = packed_block_bytes(rows_t);
  uint8_t* blocks = a.ws.bpx + (int64_t)tile * kc * bb;
  const uint8_t* rows = a.ws.xq + (int64_t)t * 2 * dp;
  const int units = kc * 8 * terms;   // (chunk, term, unit); units past d are never read by the MMAs
  for (int i0 = lane; i0 < units; i0 += 128) {
    uint4 v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = i0 + 32 * r;
      if (i < units) {
        const int c = i / (8 * terms), term = (i >> 3) % terms, u = i & 7;
        v[r] = __ldcg(reinterpret_cast<const uint4*>(rows + term * dp + c * kKChunk) + u);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = i0 + 32 * r;
      if (i < units) {
        const int c = i / (8 * terms), term = (i >> 3) % terms, u = i & 7;
        uint4* q = reinterpret_cast<uint4*>(blocks + (int64_t)c * bb + packed_unit_offset(terms * col + term, u));
        if (in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status)) *q = v[r];
      }
    }
  }
  const uint8_t* sf = a.ws.xsf + (int64_t)t * 2 * (dp / 32);
  for (int i = lane; i < terms * nb; i += 32) {
    const int term = i / nb, b = i - term * nb;
    uint8_t* q = blocks + (int64_t)(b / 4) * bb + packed_sf_offset(rows_t, terms * col + term, b);
    if (in_bounds(q, a.ws.bpx, a.ws.bpx_end, a.ws.status)) *q = __ldcg(sf + term * (dp / 32) + b);
  }
}

constexpr int64_t kPackChunkTasksMax = 1 << 16;   // up to this many (pair, chunk) tasks: one warp each

// Every pair's activation rows and scales into its token tile's packed blocks: one warp
// per (pair, 128-chunk) for small batches, one warp per pair otherwise.  FP4: MXFP4
// activations (64-byte rows of packed codes), a separate instantiation.
template <bool FP4>
__global__ void pack_kernel(FwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int P = a.T * a.k, bt = a.ws.tile_tokens, kc = a.ws.dp / kKChunk;
  if ((int64_t)P * kc > kPackChunkTasksMax) {
    for (int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < P; p += gridDim.x * (blockDim.x >> 5)) {
      const int q = a.ws.perm[p];
      const int e = a.ws.topk_idx[q];
      const int j = p - a.ws.offsets[e];
      pack_pair<FP4>(a, q / a.k, a.ws.tile_base[e] + j / bt, j % bt);
    }
    return;
  }
  const int64_t tasks = (int64_t)P * kc;
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < tasks;
       w += (int64_t)gridDim.x * (blockDim.x >> 5)) {
    const int p = (int)(w / kc), c = (int)(w - (int64_t)p * kc);
    const int q = a.ws.perm[p];
    const int e = a.ws.topk_idx[q];
    const int j = p - a.ws.offsets[e];
    pack_pair_chunk<FP4>(a, q / a.k, a.ws.tile_base[e] + j / bt, j % bt, c);
  }
}

// y[t] = bf16(x[t] + sum_j sum_s ys[s][t*k + j]), j in slot order, then split order;
// with y_partial the fp32 sum alone (no residual: one rank's slice of the intermediate
// features, summed over the ranks afterwards).
__global__ void combine_kernel(FwdArgs a) {
  pdl_trigger();
  pdl_wait();
  const int i4 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i4 >= a.d) return;
  const int64_t P = (int64_t)a.T * a.k;
  const int ksplit = a.ws.ntiles[1];   // the splits the down GEMM of this call used
  for (int t = blockIdx.y; t < a.T; t += gridDim.y) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (!a.y_partial) {
      const uint2 xr = *reinterpret_cast<const uint2*>(a.x + (int64_t)t * a.d + i4);
      v[0] = __uint_as_float(xr.x << 16);
      v[1] = __uint_as_float(xr.x & 0xFFFF0000u);
      v[2] = __uint_as_float(xr.y << 16);
      v[3] = __uint_as_float(xr.y & 0xFFFF0000u);
    }
    for (int j = 0; j < a.k; ++j) {
      const int64_t p = (int64_t)t * a.k + j;   // the down GEMM writes pair t * k + j's row there
      for (int sp = 0; sp < ksplit; ++sp) {   // partial sums of a split down GEMM
        const float4 o = *reinterpret_cast<const float4*>(a.ws.ys + (sp * P + p) * a.d + i4);
        v[0] += o.x;
        v[1] += o.y;
        v[2] += o.z;
        v[3] += o.w;
      }
    }
    if (a.y_partial) {
      *reinterpret_cast<float4*>(a.y_partial + (int64_t)t * a.d + i4) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
      uint2 out;
      out.x = (uint32_t)bf16_bits_rne(v[0]) | ((uint32_t)bf16_bits_rne(v[1]) << 16);
      out.y = (uint32_t)bf16_bits_rne(v[2]) | ((uint32_t)bf16_bits_rne(v[3]) << 16);
      *reinterpret_cast<uint2*>(a.y + (int64_t)t * a.d + i4) = out;
    }
  }
}

// ----------------------------------------------------------------------------------
// Rows that finish a block: y = bf16(x + s) and, with norm_w, the next block's RMSNorm of
// it, y_norm = bf16(y / sqrt(mean(y^2) + eps) * norm_w) on the bf16 y (each block holds two
// RMSNorms: "Transformer 块" of the ewbang.com GPT-OSS article).  s is either the sum of the
// token's k expert outputs (its k consecutive rows of ys, slot order then split order, as combine_kernel)
// or a dense fp32 row (the all-reduced partial outputs of the ranks that hold slices of the
// intermediate features).  One CTA of 256 threads per row; the row's sum of squares is a
// block reduction in fixed order.
// ----------------------------------------------------------------------------------
struct FinishArgs {
  int32_t T, d, k;
  const int32_t* ksplit;  // the splits the down GEMM of this call used (device)
  int64_t P;
  const uint16_t* x;
  const float* ys;        // pair outputs [ksplit][P][d] (or NULL)
  const int32_t* inv;
  const float* s;         // dense fp32 [T][d] (or NULL)
  const float* norm_w;    // NULL: y only
  float eps;
  uint16_t* y;
  uint16_t* y_norm;
};

constexpr int kFinishThreads = 256;

__global__ void __launch_bounds__(kFinishThreads) finish_rows_kernel(FinishArgs f) {
  __shared__ float s_red[kFinishThreads / 32];
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ks = f.ys ? *f.ksplit : 0;
  for (int t = blockIdx.x; t < f.T; t += gridDim.x) {
    float ss = 0.f;
    for (int i4 = tid * 4; i4 < f.d; i4 += kFinishThreads * 4) {
      const uint2 xr = *reinterpret_cast<const uint2*>(f.x + (int64_t)t * f.d + i4);
      float v[4] = {__uint_as_float(xr.x << 16), __uint_as_float(xr.x & 0xFFFF0000u), __uint_as_float(xr.y << 16),
                    __uint_as_float(xr.y & 0xFFFF0000u)};
      if (f.ys) {
        for (int j = 0; j < f.k; ++j) {
          const int64_t p = (int64_t)t * f.k + j;
          for (int sp = 0; sp < ks; ++sp) {
            const float4 o = *reinterpret_cast<const float4*>(f.ys + (sp * f.P + p) * f.d + i4);
            v[0] += o.x;
            v[1] += o.y;
            v[2] += o.z;
            v[3] += o.w;
          }
        }
      } else {
        const float4 o = *reinterpret_cast<const float4*>(f.s + (int64_t)t * f.d + i4);
        v[0] += o.x;
        v[1] += o.y;
        v[2] += o.z;
        v[3] += o.w;
      }
      uint16_t b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        b[q] = bf16_bits_rne(v[q]);
        const float yb = bf16_to_f32(b[q]);
        ss = fmaf(yb, yb, ss);
      }
      uint2 out;
      out.x = (uint32_t)b[0] | ((uint32_t)b[1] << 16);
      out.y = (uint32_t)b[2] | ((uint32_t)b[3] << 16);
      *reinterpret_cast<uint2*>(f.y + (int64_t)t * f.d + i4) = out;
    }
    if (f.norm_w) {
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_red[warp] = ss;
      __syncthreads();
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kFinishThreads / 32; ++w) tot += s_red[w];
      const float r = 1.0f / sqrtf(tot / (float)f.d + f.eps);
      for (int i4 = tid * 4; i4 < f.d; i4 += kFinishThreads * 4) {   // this thread's own y values
        const uint2 yr = *reinterpret_cast<const uint2*>(f.y + (int64_t)t * f.d + i4);
        const float4 g = *reinterpret_cast<const float4*>(f.norm_w + i4);
        const float v0 = __uint_as_float(yr.x << 16) * r * g.x, v1 = __uint_as_float(yr.x & 0xFFFF0000u) * r * g.y;
        const float v2 = __uint_as_float(yr.y << 16) * r * g.z, v3 = __uint_as_float(yr.y & 0xFFFF0000u) * r * g.w;
        uint2 out;
        out.x = (uint32_t)bf16_bits_rne(v0) | ((uint32_t)bf16_bits_rne(v1) << 16);
        out.y = (uint32_t)bf16_bits_rne(v2) | ((uint32_t)bf16_bits_rne(v3) << 16);
        *reinterpret_cast<uint2*>(f.y_norm + (int64_t)t * f.d + i4) = out;
      }
      __syncthreads();   // s_red is reused by the next row
    }
  }
}

// Sets a kernel's dynamic shared-memory limit once per device (the largest size asked).
template <class K>
bool ensure_smem_limit(K kern, size_t bytes, std::atomic<int>* limits /*[64]*/) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::atomic<int>& lim = limits[dev & 63];
  if ((int)bytes <= lim.load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
    return false;
  int cur = lim.load();
  while ((int)bytes > cur && !lim.compare_exchange_weak(cur, (int)bytes)) {
  }
  return true;
}

template <int NJ>
int launch_route_nj(const FwdArgs& a) {
  static std::atomic<int> tok_limits[64], tile_limits[64], tile_limits_fp4[64];
  if (a.T <= kTokenKernelMaxT) {
    const size_t smem = sizeof(float) * (a.d + 32 * NJ);
    if (!ensure_smem_limit(route_token_kernel<NJ>, smem, tok_limits)) return -1;
    ev_before(a);
    if (launch_kernel_cluster(route_token_kernel<NJ>, dim3(a.T * kTokCluster), dim3(kTokThreads), smem, a.stream,
                              false, (unsigned)kTokCluster, a) != cudaSuccess)
      return -1;
    ev_after(a);
    return 1;
  }
  // the tensor-core router keeps one CTA per 128 tokens busy for the whole reduction axis:
  // it wins from about half the SMs (8192 tokens x 128 experts: 0.27 ms against 0.32 ms;
  // 16384: 0.30 against 0.55); below that the 16-token tiles spread further (4096 tokens
  // x 32 experts: 0.09 ms against 0.23 ms)
  if ((a.T + 127) / 128 >= kRouteMmaMinCtas && route_mma_fits(a.E, a.d)) return launch_route_mma(a);
  // chunk width and stages: the router rows of a stage stay within shared memory (up to 128
  // experts: 64-wide chunks; 128 experts take two stages of 34 KB, which measured faster
  // than four stages of 32-wide chunks)
  constexpr int RKC = NJ <= 4 ? 64 : 32;
  constexpr int NSC = NJ == 4 ? 2 : 4;
  using C = RouteTilesCfg<NJ, RKC, NSC>;
  const size_t smem = C::smem(a.d);
  auto kern = a.ws.fp4 ? route_tiles_kernel<NJ, RKC, NSC, true> : route_tiles_kernel<NJ, RKC, NSC, false>;
  if (!ensure_smem_limit(kern, smem, a.ws.fp4 ? tile_limits_fp4 : tile_limits)) return -1;
  ev_before(a);
  kern<<<(a.T + kRT - 1) / kRT, 256, smem, a.stream>>>(a);
  ev_after(a);
  return 1;
}

}  // namespace

int launch_quantize(const float* w, int32_t E, int32_t N, int32_t K, int32_t role, uint8_t* codes,
                    uint8_t* scales, int32_t* status, cudaStream_t st) {
  const int64_t Kp = kpad128(K);
  // padding (rows past N, k past K): codes 0, scale bytes 127 (2^0)
  const size_t blocks = (size_t)E * ((N + 127) / 128) * (Kp / kKChunk);
  if (Kp != K || N % 128) {
    if (cudaMemsetAsync(codes, 0, blocks * kCodeBlockBytes, st) != cudaSuccess) return -1;
    if (cudaMemsetAsync(scales, 127, blocks * kSfGroupBytes, st) != cudaSuccess) return -1;
  }
  const int64_t nblocks = (int64_t)E * N * (K / 32);
  const int64_t want = (nblocks + 7) / 8;
  const int grid = (int)std::min<int64_t>(want, 148 * 64);
  quantize_kernel<<<grid, 256, 0, st>>>(w, nblocks, N, K, role, codes, scales, status,
                                        codes + blocks * kCodeBlockBytes, scales + blocks * kSfGroupBytes);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_route(const FwdArgs& a_in) {
  const int tile_tokens = a_in.ws.tile_tokens;
  int n = 0;
  FwdArgs a = a_in;
  // fuse_group carries the token-tile size into the routing kernel (0 = separate kernels)
  a.fuse_group = a_in.fuse_group ? tile_tokens : 0;
  const size_t clear_ints = (size_t)a.E + 4 + (a.fuse_combine ? (size_t)a.T * ((a.d + 127) / 128) : 0);
  if (cudaMemsetAsync(a.ws.counts, 0, sizeof(int32_t) * clear_ints, a.stream) != cudaSuccess) return -1;
  int r;
  if (a.E <= 32) r = launch_route_nj<1>(a);
  else if (a.E <= 64) r = launch_route_nj<2>(a);
  else if (a.E <= 128) r = launch_route_nj<4>(a);
  else r = launch_route_nj<8>(a);
  if (r < 0) return -1;
  n += r;
  if (!a.fuse_group) {
    ev_before(a);
    if (launch_kernel(group_kernel, dim3(a.E), dim3(1024), 0, a.stream, a.pdl != 0, a, tile_tokens) != cudaSuccess)
      return -1;
    ev_after(a);
    ++n;
  }
  const int64_t P = (int64_t)a.T * a.k, tasks = P * (a.ws.dp / kKChunk);
  const int64_t warps = tasks > kPackChunkTasksMax ? P : tasks;   // one warp per task (pack_kernel)
  ev_before(a);
  if (launch_kernel(a.ws.fp4 ? pack_kernel<true> : pack_kernel<false>,
                    dim3((unsigned)std::min<int64_t>((warps + 7) / 8, 148 * 32)), dim3(256), 0, a.stream, a.pdl != 0,
                    a) != cudaSuccess)
    return -1;
  ev_after(a);
  ++n;
  return cudaGetLastError() == cudaSuccess ? n : -1;
}

int launch_combine(const FwdArgs& a) {
  if (a.next_norm_w) {   // y and the next block's RMSNorm of it: whole rows per CTA
    FinishArgs f{};
    f.T = a.T;
    f.d = a.d;
    f.k = a.k;
    f.ksplit = a.ws.ntiles + 1;
    f.P = (int64_t)a.T * a.k;
    f.x = a.x;
    f.ys = a.ws.ys;
    f.inv = a.ws.inv;
    f.norm_w = a.next_norm_w;
    f.eps = a.next_eps;
    f.y = a.y;
    f.y_norm = a.y_norm;
    ev_before(a);
    if (launch_kernel(finish_rows_kernel, dim3((unsigned)std::min(a.T, 148 * 8)), dim3(kFinishThreads), 0, a.stream,
                      a.pdl != 0, f) != cudaSuccess)
      return -1;
    ev_after(a);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
  }
  dim3 grid((a.d / 4 + 127) / 128, std::min(a.T, 65535));
  ev_before(a);
  if (launch_kernel(combine_kernel, grid, dim3(128), 0, a.stream, a.pdl != 0, a) != cudaSuccess) return -1;
  ev_after(a);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_residual_norm(int32_t T, int32_t d, const uint16_t* x, const float* s, const float* norm_w, float eps,
                         uint16_t* y, uint16_t* y_norm, cudaStream_t st) {
  FinishArgs f{};
  f.T = T;
  f.d = d;
  f.x = x;
  f.s = s;
  f.norm_w = norm_w;
  f.eps = eps;
  f.y = y;
  f.y_norm = y_norm;
  if (launch_kernel(finish_rows_kernel, dim3((unsigned)std::min(T, 148 * 8)), dim3(kFinishThreads), 0, st, false,
                    f) != cudaSuccess)
    return -1;
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace moe
