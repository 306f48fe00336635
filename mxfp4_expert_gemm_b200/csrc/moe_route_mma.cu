// Router for large batches on the tensor cores: RMSNorm, router logits, top-k + softmax,
// and the expert GEMMs' activation format of xe = bf16(RMSNorm(x)), 128 tokens per CTA.
//
// Layer definition (web pages on gpt-oss): RMSNorm per "From GPT-2 to gpt-oss" sec. 7
// (divide by the RMS; rms_norm_eps 1e-5 from the llm-atlas GPT-OSS 20B config table); the
// router of the ewbang.com GPT-OSS article, section 混合专家模型 (a small network scores the
// experts; several are chosen per token and weighted).
//
// The logits l = W_r . xn (xn the unrounded fp32 RMSNorm output) are an M = 128 tokens x
// N = E experts x K = d product.  They decide the top-k, so they must stay at fp32
// accuracy: each operand is split into a TF32 part and a TF32 remainder (hi = tf32(v),
// lo = tf32(v - hi)) and the tensor cores accumulate hi.hi + hi.lo + lo.hi in fp32 (the
// dropped lo.lo term is below 2^-20 of a product).
//
// Per CTA: a first pass over its tokens' rows gives 1 / rms per token.  The reduction axis
// is then walked in chunks of 32 (one 128-byte row of 32 fp32 per token and per expert, one
// 32-value block of the activation format) through a two-stage ring: the threads load a
// chunk of x and of W_r, normalize x, write the TF32 parts into 128B-swizzled K-major
// tiles, and write xe's activation-format terms for the expert GEMMs (two E4M3 terms, the
// MXFP8 term or MXFP4 codes, with their block scales); one elected thread issues the 12
// MMAs of the chunk (4 K-steps x 3 products) and commits them to the stage's barrier.  The
// accumulator [128 tokens][E] is read back from TMEM into shared memory and each warp runs
// the top-k + softmax of 16 tokens (the same routine as the other routers).
#include <cuda.h>
#include <algorithm>
#include <atomic>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kRM = 128;          // tokens per CTA (MMA M)
constexpr int kRK = 32;           // reduction chunk: 32 fp32 per row, one 32-value block
constexpr int kRThreads = 512;   // 16 warps: the per-chunk conversions are latency-bound chains
constexpr int kXItems = kRM * 4 / kRThreads;   // activation items (8 values) per thread and chunk
constexpr uint64_t kRWaitNs = 2000000000ull;

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Byte offset of 16-byte unit u (of 8) of row r in a 128B-swizzled K-major tile.
__device__ __forceinline__ int sw128(int r, int u) { return r * 128 + ((u ^ (r & 7)) << 4); }

struct RouteMmaLayout {
  int N;            // MMA N: E rounded up to 16
  int a_stage;      // bytes of one stage of A (hi then lo)
  int b_half;       // bytes of one B part (N rows x 128)
  int b_stage;      // bytes of one stage of B (hi then lo)
  int ring;         // two stages of A and B
  int logit_ld;     // floats per row of the logits staged after the GEMM
  int gamma_off;    // RMSNorm weights [d] follow the ring
  size_t smem;
};

inline RouteMmaLayout route_mma_layout(int E, int d, int NJ) {
  RouteMmaLayout L;
  L.N = std::max(16, (E + 15) / 16 * 16);
  L.a_stage = 2 * kRM * 128;
  L.b_half = L.N * 128;
  L.b_stage = 2 * L.b_half;
  L.ring = 2 * (L.a_stage + L.b_stage);
  L.logit_ld = 32 * NJ + 1;
  const int logits = kRM * L.logit_ld * 4;
  L.gamma_off = std::max(L.ring, logits);
  L.smem = (size_t)L.gamma_off + 4 * (size_t)d + 1024;
  return L;
}

template <int NJ, int FMT>   // FMT: 0 bf16 (two E4M3 terms), 1 MXFP8, 2 MXFP4
__global__ void __launch_bounds__(kRThreads, 1) route_mma_kernel(FwdArgs a, RouteMmaLayout L) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_g = reinterpret_cast<float*>(smem + L.gamma_off);
  __shared__ float s_r[kRM];
  __shared__ uint64_t mma_done[2];
  __shared__ uint32_t s_tmem;
  pdl_trigger();
  const int E = a.E, d = a.d, dp = a.ws.dp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRM;
  const int nt = min(kRM, a.T - t0);
  const int nch = d / kRK;
  const uint32_t tmem_cols = L.N <= 32 ? 32 : L.N <= 64 ? 64 : L.N <= 128 ? 128 : 256;
  auto A_hi = [&](int s) { return smem + s * L.a_stage; };
  auto B_hi = [&](int s) { return smem + 2 * L.a_stage + s * L.b_stage; };

  if (tid == 0) {
    ptx::mbar_init(&mma_done[0], 1);
    ptx::mbar_init(&mma_done[1], 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, tmem_cols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  // B rows E..N-1 stay zero (both stages, both parts); gamma into shared memory
  for (int i = tid; i < 2 * 2 * (L.N - E) * 32; i += kRThreads) {
    const int part = i / ((L.N - E) * 32), rem = i % ((L.N - E) * 32);
    reinterpret_cast<float*>(smem + 2 * L.a_stage + (part >> 1) * L.b_stage + (part & 1) * L.b_half +
                             E * 128)[rem] = 0.f;
  }
  for (int i = tid * 4; i < d; i += kRThreads * 4)
    *reinterpret_cast<float4*>(s_g + i) = *reinterpret_cast<const float4*>(a.norm_w + i);
  // 1 / rms of the CTA's tokens: warp w takes tokens kRows w .. kRows w + kRows - 1, the
  // loads of all its rows at one column step in flight together (each token's sum keeps its order: lane
  // partial sums over the row, then the warp reduction)
  {
    constexpr int kRows = kRM / (kRThreads / 32);   // tokens per warp
    float ss[kRows];
#pragma unroll
    for (int q = 0; q < kRows; ++q) ss[q] = 0.f;
    for (int i = lane * 8; i < d; i += 256) {
      uint4 v[kRows];
#pragma unroll
      for (int q = 0; q < kRows; ++q) {
        const int m = kRows * warp + q;
        v[q] = (m < nt) ? __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)(t0 + m) * d + i))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int q = 0; q < kRows; ++q) {
        const uint32_t wv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = __uint_as_float(wv[j] << 16), hi = __uint_as_float(wv[j] & 0xFFFF0000u);
          ss[q] = fmaf(lo, lo, ss[q]);
          ss[q] = fmaf(hi, hi, ss[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kRows; ++q) {
      float t = ss[q];
#pragma unroll
      for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      const int m = kRows * warp + q;
      if (lane == 0) s_r[m] = m < nt ? 1.0f / sqrtf(t / (float)d + a.eps) : 0.f;
    }
  }
  ptx::fence_proxy_async_smem();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t idesc = ptx::idesc_tf32(kRM, L.N);

  // Raw loads of one chunk: x items (token m = i / 4, 8 values at 8 (i % 4)) for
  // i = tid + kRThreads p; W_r units (row e = j / 8, 4 values at 4 (j % 8)) for
  // j = tid + kRThreads r.
  constexpr int kWU = NJ * 32 * 8 / kRThreads > 0 ? NJ * 32 * 8 / kRThreads : 1;   // W units per thread
  // Three register buffers of raw loads, two chunks in flight while one is converted
  // (the loop is unrolled by three so that every buffer keeps a fixed register name)
  struct Raw {
    uint4 x[kXItems];
    float4 w[kWU];
  };
  auto load_chunk = [&](Raw& rb, int c) {
    const int k0 = c * kRK;
#pragma unroll
    for (int p = 0; p < kXItems; ++p) {
      const int i = tid + kRThreads * p, m = i >> 2, g = i & 3;
      rb.x[p] = (m < nt) ? __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)(t0 + m) * d + k0 + 8 * g))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int r = 0; r < kWU; ++r) {
      const int j = tid + kRThreads * r, e = j >> 3, u = j & 7;
      rb.w[r] = (e < E) ? __ldg(reinterpret_cast<const float4*>(a.router_w + (int64_t)e * d + k0 + 4 * u))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };

  bool ok = true;
  volatile int no_abort = 0;   // (the bounded waits' abort flag: unused here)
  int issued = -1;             // the last chunk whose MMAs were committed
  // One chunk: convert it into stage c % 2 and issue its MMAs.  False when a wait gave up.
  auto process = [&](int c, const Raw& cur) -> bool {
    const int s = c & 1, k0 = c * kRK;
    // the MMAs that read this stage two chunks ago are done
    if (c >= 2) ok = ptx::mbar_wait_bounded(&mma_done[s], (uint32_t)((c - 2) >> 1) & 1, &no_abort, kRWaitNs);
    if (!__syncthreads_and(ok)) return false;
    // ---- activations: TF32 parts into A, the activation format into xq / xsf
#pragma unroll
    for (int p = 0; p < kXItems; ++p) {
      const int i = tid + kRThreads * p, m = i >> 2, g = i & 3;
      const float r = s_r[m];
      const uint32_t w4[4] = {cur.x[p].x, cur.x[p].y, cur.x[p].z, cur.x[p].w};
      float xn[8], hi[8], lo[8], xe[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float xv = (j & 1) ? __uint_as_float(w4[j >> 1] & 0xFFFF0000u) : __uint_as_float(w4[j >> 1] << 16);
        xn[j] = xv * r * s_g[k0 + 8 * g + j];
        hi[j] = ptx::to_tf32(xn[j]);
        lo[j] = ptx::to_tf32(xn[j] - hi[j]);
        xe[j] = bf16f(bf16_bits_rne(xn[j]));
      }
      uint8_t* ah = A_hi(s);
      uint8_t* al = ah + kRM * 128;
      *reinterpret_cast<float4*>(ah + sw128(m, 2 * g)) = make_float4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<float4*>(ah + sw128(m, 2 * g + 1)) = make_float4(hi[4], hi[5], hi[6], hi[7]);
      *reinterpret_cast<float4*>(al + sw128(m, 2 * g)) = make_float4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<float4*>(al + sw128(m, 2 * g + 1)) = make_float4(lo[4], lo[5], lo[6], lo[7]);
      // the 32-value block of token m is held by 4 consecutive lanes (8 values each)
      const bool live = m < nt;
      uint8_t* xq = a.ws.xq + (int64_t)(t0 + m) * 2 * dp;
      uint8_t* sf = a.ws.xsf + (int64_t)(t0 + m) * 2 * (dp / 32);
      if (FMT == 2) {
        uint32_t codes, s1;
        e2m1_quant<8>(xe, codes, s1);
        if (live) {
          *reinterpret_cast<uint32_t*>(xq + (k0 + 8 * g) / 2) = codes;
          if (g == 0) sf[k0 / 32] = (uint8_t)s1;
        }
      } else {
        uint32_t hi2[2], lo2[2], s1, s2;
        {
          const float v0[4] = {xe[0], xe[1], xe[2], xe[3]};
          const float v1[4] = {xe[4], xe[5], xe[6], xe[7]};
          // one block over 4 lanes x 8 values: the split's amax reduction runs over the 8
          // values and the 4 lanes; done as two halves of 4 values sharing one block scale
          float amax = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(xe[j]));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
          const int e1 = e4m3_block_exp(amax), e2 = e1 - 4;
          const float inv1 = pow2f(-e1), sc1 = pow2f(e1), inv2 = pow2f(-e2);
          uint32_t h0 = 0u, h1 = 0u, l0 = 0u, l1 = 0u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t q0 = e4m3x2(v0[j] * inv1, 0.f) & 0xFFu, q1 = e4m3x2(v1[j] * inv1, 0.f) & 0xFFu;
            h0 |= q0 << (8 * j);
            h1 |= q1 << (8 * j);
            l0 |= (e4m3x2((v0[j] - e4m3_to_f32(q0) * sc1) * inv2, 0.f) & 0xFFu) << (8 * j);
            l1 |= (e4m3x2((v1[j] - e4m3_to_f32(q1) * sc1) * inv2, 0.f) & 0xFFu) << (8 * j);
          }
          hi2[0] = h0; hi2[1] = h1; lo2[0] = l0; lo2[1] = l1;
          s1 = (uint32_t)(e1 + 127);
          s2 = (uint32_t)(e2 + 127);
        }
        if (live) {
          *reinterpret_cast<uint2*>(xq + k0 + 8 * g) = make_uint2(hi2[0], hi2[1]);
          if (FMT == 0) *reinterpret_cast<uint2*>(xq + dp + k0 + 8 * g) = make_uint2(lo2[0], lo2[1]);
          if (g == 0) {
            sf[k0 / 32] = (uint8_t)s1;
            if (FMT == 0) sf[dp / 32 + k0 / 32] = (uint8_t)s2;
          }
        }
      }
    }
    // ---- router weights: TF32 parts into B
#pragma unroll
    for (int r = 0; r < kWU; ++r) {
      const int j = tid + kRThreads * r, e = j >> 3, u = j & 7;
      if (e < E) {
        const float4 w = cur.w[r];
        const float4 h = make_float4(ptx::to_tf32(w.x), ptx::to_tf32(w.y), ptx::to_tf32(w.z), ptx::to_tf32(w.w));
        const float4 l = make_float4(ptx::to_tf32(w.x - h.x), ptx::to_tf32(w.y - h.y), ptx::to_tf32(w.z - h.z),
                                     ptx::to_tf32(w.w - h.w));
        *reinterpret_cast<float4*>(B_hi(s) + sw128(e, u)) = h;
        *reinterpret_cast<float4*>(B_hi(s) + L.b_half + sw128(e, u)) = l;
      }
    }
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (warp == 0) {
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        const uint64_t ah = ptx::smem_desc_k_sw128(A_hi(s)), al = ptx::smem_desc_k_sw128(A_hi(s) + kRM * 128);
        const uint64_t bh = ptx::smem_desc_k_sw128(B_hi(s)), bl = ptx::smem_desc_k_sw128(B_hi(s) + L.b_half);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {   // K = 8 per MMA: 32 bytes of each row
          ptx::mma_tf32_ss(tmem, ah + 2 * ks, bh + 2 * ks, idesc, (c | ks) != 0);
          ptx::mma_tf32_ss(tmem, ah + 2 * ks, bl + 2 * ks, idesc, 1u);
          ptx::mma_tf32_ss(tmem, al + 2 * ks, bh + 2 * ks, idesc, 1u);
        }
        ptx::tc_commit(&mma_done[s]);
      }
      __syncwarp();
    }
    issued = c;
    return true;
  };
  Raw r0, r1, r2;
  load_chunk(r0, 0);
  if (nch > 1) load_chunk(r1, 1);
  for (int c = 0; c < nch; c += 3) {
    if (c + 2 < nch) load_chunk(r2, c + 2);
    if (!process(c, r0) || c + 1 >= nch) break;
    if (c + 3 < nch) load_chunk(r0, c + 3);
    if (!process(c + 1, r1) || c + 2 >= nch) break;
    if (c + 4 < nch) load_chunk(r1, c + 4);
    if (!process(c + 2, r2)) break;
  }
  // the last committed chunk's MMAs (and with them all earlier ones) are done
  if (issued >= 0) {
    no_abort = 0;
    const bool drained = ptx::mbar_wait_bounded(&mma_done[issued & 1], (uint32_t)(issued >> 1) & 1, &no_abort,
                                                kRWaitNs);
    ok = ok && drained;
  }
  ok = __syncthreads_and(ok) && issued == nch - 1;
  ptx::tc_fence_after();
  if (ok) {
    // ---- logits [128 tokens][E] from TMEM (warp q reads lanes 32q..32q+31) into shared memory
    float* s_l = reinterpret_cast<float*>(smem);
    if (warp < 4) {
      const int m = 32 * warp + lane;
      for (int c0 = 0; c0 < 32 * NJ; c0 += 32) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) s_l[m * L.logit_ld + c0 + j] = __uint_as_float(v[j]);
      }
    }
    __syncthreads();
    // ---- top-k + softmax: warp w takes tokens kTokPerWarp w .. kTokPerWarp (w + 1) - 1
    constexpr int kTokPerWarp = kRM / (kRThreads / 32);
    for (int m = kTokPerWarp * warp; m < kTokPerWarp * (warp + 1) && m < nt; ++m) {
      float l[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        l[j] = (e < E) ? s_l[m * L.logit_ld + e] + (a.router_b ? a.router_b[e] : 0.f) : -INFINITY;
      }
      warp_topk_softmax<NJ>(l, E, a.k, t0 + m, a);
    }
  } else if (tid == 0) {
    set_status(a.ws.status, MOE_ERR_TIMEOUT);
  }
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, tmem_cols);
  }
}

template <int NJ, int FMT>
int launch_nj_fmt(const FwdArgs& a) {
  static std::atomic<int> limits[64];
  const RouteMmaLayout L = route_mma_layout(a.E, a.d, NJ);
  auto kern = route_mma_kernel<NJ, FMT>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::atomic<int>& lim = limits[dev & 63];
  if ((int)L.smem > lim.load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem) != cudaSuccess) return -1;
    lim.store((int)L.smem, std::memory_order_release);
  }
  ev_before(a);
  kern<<<(a.T + kRM - 1) / kRM, kRThreads, L.smem, a.stream>>>(a, L);
  ev_after(a);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

template <int NJ>
int launch_nj(const FwdArgs& a) {
  if (a.ws.fp4) return launch_nj_fmt<NJ, 2>(a);
  return a.ws.terms == 1 ? launch_nj_fmt<NJ, 1>(a) : launch_nj_fmt<NJ, 0>(a);
}

}  // namespace

bool route_mma_fits(int E, int d) {
  const int NJ = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8;
  return route_mma_layout(E, d, NJ).smem <= 227 * 1024;
}

int launch_route_mma(const FwdArgs& a) {
  if (a.E <= 32) return launch_nj<1>(a);
  if (a.E <= 64) return launch_nj<2>(a);
  if (a.E <= 128) return launch_nj<4>(a);
  return launch_nj<8>(a);
}

}  // namespace moe
