// CUDA-core (fp32 FMA) expert MLPs over the token tiles of the grouping step.
//
// A plain tiled implementation of the SwiGLU expert ("From GPT-2 to gpt-oss",
// sec. 3: three linears, silu gate; swiglu_limit 7 from the llm-atlas config
// table) on MXFP4 weights (ewbang.com GPT-OSS article, section 量化).  It has no
// range limits and no tensor cores; the library keeps it as an independent
// cross-check of the tcgen05 paths (MOE_PATH_SIMT).
#include <cuda_fp16.h>
#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int ST = 64;  // token rows per tile (the grouping step's tile size for this path)
constexpr int SJ = 32;  // output columns per CTA
constexpr int SK = 32;  // K per step: one MXFP4 block

__device__ __forceinline__ float e2m1_f32(int c) {
  const float mag = (c & 6) ? __int_as_float((((c >> 1) & 3) + 126) << 23) * (1.0f + 0.5f * (c & 1))
                            : 0.5f * (c & 1);
  return (c & 8) ? -mag : mag;
}

// Decode one 32-value block of row `row` of expert `e` (library MXFP4 layout).
__device__ __forceinline__ void decode_block(const uint8_t* codes, const uint8_t* scales, int e, int64_t row,
                                             int64_t N, int K, int kb, float* out, int out_stride,
                                             int32_t* status) {
  const uint4 q = *reinterpret_cast<const uint4*>(codes + mx_code_chunk_offset(e, row, kb, N, K));
  const int sb = scales[mx_scale_offset(e, row, kb, N, K)];
  if (sb == 0xFF) set_status(status, MOE_ERR_NONFINITE);
  const float sc = ldexpf(1.0f, sb - 127);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int c = (w[i >> 3] >> (4 * (i & 7))) & 15;
    out[i * out_stride] = e2m1_f32(c) * sc;
  }
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// h[p][j] = bf16(silu(min(g, L)) * clamp(u, -L, L)), g/u = W1 gate/up rows . xs[p]
__global__ void __launch_bounds__(256) gate_up_simt(FwdArgs a) {
  __shared__ float s_a[SK][ST + 1];
  __shared__ float s_g[SK][SJ + 1];
  __shared__ float s_u[SK][SJ + 1];
  if ((int)blockIdx.x >= a.ws.ntiles[0]) return;
  const Tile tl = a.ws.tiles[blockIdx.x];
  const int d = a.d, I = a.I;
  const int j0 = blockIdx.y * SJ;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float ag[4][2] = {}, au[4][2] = {};
  for (int kb = 0; kb < d / SK; ++kb) {
    {  // activations: 64 rows x 32 k (f16), 8 per thread
      const int r = tid / 4, c8 = (tid % 4) * 8;
      float v[8] = {};
      if (r < tl.rows) {
        const uint4 q = *reinterpret_cast<const uint4*>(a.ws.xs + (int64_t)(tl.row0 + r) * d + kb * SK + c8);
        const __half2* hp = reinterpret_cast<const __half2*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(hp[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) s_a[c8 + i][r] = v[i];
    }
    if (tid < 2 * SJ) {  // weights: 32 gate rows + 32 up rows, one block each
      const int jj = tid % SJ;
      const int64_t row = (tid < SJ) ? (j0 + jj) : (I + j0 + jj);
      decode_block(a.w1c, a.w1s, tl.e, row, 2 * I, d, kb, (tid < SJ) ? &s_g[0][jj] : &s_u[0][jj], SJ + 1,
                   a.ws.status);
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SK; ++kk) {
      float av[4], gv[2], uv[2];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = s_a[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        gv[j] = s_g[kk][tx * 2 + j];
        uv[j] = s_u[kk][tx * 2 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          ag[i][j] = fmaf(av[i], gv[j], ag[i][j]);
          au[i][j] = fmaf(av[i], uv[j], au[i][j]);
        }
    }
    __syncthreads();
  }
  const float L = a.limit;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= tl.rows) continue;
    uint16_t hv[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float g = fminf(ag[i][j], L);
      const float u = fminf(fmaxf(au[i][j], -L), L);
      const float hval = g / (1.0f + expf(-g)) * u;
      const uint16_t hb = f32_to_bf16_rne(hval);
      hv[j] = __half_as_ushort(__float2half_rn(__uint_as_float((uint32_t)hb << 16)));
    }
    *reinterpret_cast<uint32_t*>(a.ws.h + (int64_t)(tl.row0 + r) * I + j0 + tx * 2) =
        (uint32_t)hv[0] | ((uint32_t)hv[1] << 16);
  }
}

// ys[p][m] = w_sorted[p] * (W2[m] . h[p])
__global__ void __launch_bounds__(256) down_simt(FwdArgs a) {
  __shared__ float s_a[SK][ST + 1];
  __shared__ float s_w[SK][SJ + 1];
  if ((int)blockIdx.x >= a.ws.ntiles[0]) return;
  const Tile tl = a.ws.tiles[blockIdx.x];
  const int d = a.d, I = a.I;
  const int m0 = blockIdx.y * SJ;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float acc[4][2] = {};
  for (int kb = 0; kb < I / SK; ++kb) {
    {
      const int r = tid / 4, c8 = (tid % 4) * 8;
      float v[8] = {};
      if (r < tl.rows) {
        const uint4 q = *reinterpret_cast<const uint4*>(a.ws.h + (int64_t)(tl.row0 + r) * I + kb * SK + c8);
        const __half2* hp = reinterpret_cast<const __half2*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(hp[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) s_a[c8 + i][r] = v[i];
    }
    if (tid < SJ) {
      const int m = m0 + tid;
      if (m < d) decode_block(a.w2c, a.w2s, tl.e, m, d, I, kb, &s_w[0][tid], SJ + 1, a.ws.status);
      else
        for (int i = 0; i < SK; ++i) s_w[i][tid] = 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SK; ++kk) {
      float av[4], wv[2];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = s_a[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 2; ++j) wv[j] = s_w[kk][tx * 2 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= tl.rows) continue;
    const int p = tl.row0 + r;
    const float wgt = a.ws.w_sorted[p];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int m = m0 + tx * 2 + j;
      if (m < d) a.ws.ys[(int64_t)p * d + m] = wgt * acc[i][j];
    }
  }
}

}  // namespace

int launch_experts_simt(const FwdArgs& a) {
  const int P = a.T * a.k;
  const int max_tiles = (P + ST - 1) / ST + a.E;
  ev_before(a);
  gate_up_simt<<<dim3(max_tiles, a.I / SJ), 256, 0, a.stream>>>(a);
  ev_after(a);
  ev_before(a);
  down_simt<<<dim3(max_tiles, (a.d + SJ - 1) / SJ), 256, 0, a.stream>>>(a);
  ev_after(a);
  return cudaGetLastError() == cudaSuccess ? 2 : -1;
}

int simt_tile_tokens() { return ST; }

}  // namespace moe
