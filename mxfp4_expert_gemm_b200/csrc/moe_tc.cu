// tcgen05 grouped expert GEMMs: gate_up with the clamped-SwiGLU epilogue, and down
// with the routing-weight epilogue.
//
// Layer definition: the SwiGLU expert of "From GPT-2 to gpt-oss" (新智元
// translation), sec. 3 (three linears, silu(z) = z * sigmoid(z)), with
// swiglu_limit 7 from the llm-atlas GPT-OSS 20B config table; MXFP4 weights per the
// ewbang.com GPT-OSS article, section 量化 (E2M1 values, one E8M0 scale per 32).
//
// One CTA computes a 128 (weight rows) x BN (tokens of one expert) tile over the
// whole reduction axis.  The weights are the MMA's A operand and live in TMEM:
//   warp 0      TMA producer: activations [BN x 64] (128B swizzle), packed codes
//               [128 rows x 32 B] (32B swizzle) and scale bytes per 64-wide K step;
//   warp 1      TMEM allocation and the MMA issuer (one thread);
//   warps 2..5  decode: each thread owns one weight row (its TMEM lane), turns 32
//               code bytes into 64 f16 values (E2M1 -> f16 convert, times the exact
//               power-of-two scale) and stores them to the stage's TMEM columns;
//               afterwards the same warps run the epilogue.
// The decoded weights never touch shared memory, so the tensor core's shared-memory
// reads are the activations only.
//
// Gate_up tiles hold 64 gate rows (TMEM lanes 0..63) and the 64 matching up rows
// (lanes 64..127), so g and u of one output column meet in the epilogue.
#include <cuda.h>
#include <cuda_fp16.h>
#include <algorithm>
#include <mutex>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;            // weight rows per tile (TMEM lanes)
constexpr int kBK = 64;             // K per pipeline stage
constexpr int kThreads = 192;       // 6 warps
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: a stuck pipeline, not a slow one

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct TcParams {
  const Tile* tiles;
  const int32_t* ntiles;
  const uint8_t* codes;   // MXFP4 codes of W1 or W2 (library block layout)
  const uint8_t* scales;
  int32_t N;              // weight rows per expert (2I or d)
  const float* w_sorted;
  uint16_t* h_out;   // gate_up: [P][I] f16
  float* ys_out;     // down:    [P][d] f32
  int32_t* status;
  int32_t K;         // reduction length (d for gate_up, I for down)
  int32_t I, d;
  float limit;
};

template <int BN, int STAGES>
struct Cfg {
  static constexpr int ACT_BYTES = BN * 128;
  static constexpr int CODE_BYTES = kBM * 32;
  static constexpr int SCALE_BYTES = 256;
  static constexpr int STAGE_BYTES = ((ACT_BYTES + CODE_BYTES + SCALE_BYTES + 1023) / 1024) * 1024;
  static constexpr int A0 = BN < 32 ? 32 : ((BN + 31) / 32) * 32;  // first TMEM column of the A stages
  static constexpr int COLS_NEEDED = A0 + 32 * STAGES;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 32 ? 32 : COLS_NEEDED <= 64 ? 64 : COLS_NEEDED <= 128 ? 128
                                   : COLS_NEEDED <= 256 ? 256 : 512;

  // At most 512 / TMEM_COLS CTAs can hold TMEM on one SM; ask for enough shared memory
  // that no more than that become resident (a third CTA would only wait in tcgen05.alloc).
  static constexpr int SMEM_USED = STAGES * STAGE_BYTES + 1024 /*align slack*/ + 256 /*barriers*/;
  static constexpr int SMEM_FLOOR = TMEM_COLS >= 256 ? 80 * 1024 : 0;
  static constexpr int SMEM_BYTES = SMEM_USED > SMEM_FLOOR ? SMEM_USED : SMEM_FLOOR;
  static_assert(COLS_NEEDED <= 512, "TMEM budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M = 128");
};

// f16 bit pattern of 2^e, or 0 when E2M1 * 2^e is not exact in f16 (e outside [-23, 13]).
__device__ __forceinline__ uint32_t f16_pow2_bits(int e) {
  if (e > 13 || e < -23) return 0u;
  if (e >= -14) return (uint32_t)(e + 15) << 10;   // normal
  return 1u << (e + 24);                            // subnormal 2^-15 .. 2^-23
}

template <int MODE, int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    tc_expert_kernel(const __grid_constant__ CUtensorMap tm_act, const TcParams p) {
  using C = Cfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  if ((int)blockIdx.x >= *p.ntiles) return;  // uniform: more CTAs are launched than tiles exist

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* afull = full + STAGES;
  uint64_t* empty = afull + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Tile tl = p.tiles[blockIdx.x];
  const int nk = p.K / kBK;
  const int row_tile0 = (MODE == MODE_GATE_UP) ? blockIdx.y * 64 : blockIdx.y * kBM;
  // The tile's two 64-row halves: gate_up pairs gate rows j0.. with up rows I+j0..;
  // down takes rows m0..m0+63 and m0+64..m0+127 (the second half may not exist).
  const int rbA = row_tile0 / kBlkRows;
  const int rbB = (MODE == MODE_GATE_UP) ? (p.I + row_tile0) / kBlkRows : rbA + 1;
  const bool halfB = rbB < p.N / kBlkRows;
  const uint32_t tx_bytes = C::ACT_BYTES + (halfB ? 2 : 1) * (kBlkCodeBytes + kBlkScaleBytes);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&afull[s], 128);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accf, 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tm_act);
  }
  if (warp == 1) {
    ptx::tmem_alloc(s_tmem, C::TMEM_COLS);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;

  auto act_s = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto code_s = [&](int s) { return smem + s * C::STAGE_BYTES + C::ACT_BYTES; };
  auto scale_s = [&](int s) { return smem + s * C::STAGE_BYTES + C::ACT_BYTES + C::CODE_BYTES; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (kb >= STAGES && !ptx::mbar_wait_bounded(&empty[s], ((kb / STAGES) - 1) & 1, s_abort, kWaitLimitNs))
          break;
        ptx::mbar_arrive_expect_tx(&full[s], tx_bytes);
        ptx::tma_load_2d(act_s(s), &tm_act, kb * kBK, tl.row0, &full[s]);
        const int64_t bA = mx_block_index(tl.e, rbA, kb, p.N, p.K);
        ptx::bulk_load(code_s(s), p.codes + bA * kBlkCodeBytes, kBlkCodeBytes, &full[s]);
        ptx::bulk_load(scale_s(s), p.scales + bA * kBlkScaleBytes, kBlkScaleBytes, &full[s]);
        if (halfB) {
          const int64_t bB = mx_block_index(tl.e, rbB, kb, p.N, p.K);
          ptx::bulk_load(code_s(s) + kBlkCodeBytes, p.codes + bB * kBlkCodeBytes, kBlkCodeBytes, &full[s]);
          ptx::bulk_load(scale_s(s) + kBlkScaleBytes, p.scales + bB * kBlkScaleBytes, kBlkScaleBytes, &full[s]);
        }
        issued = kb + 1;
      }
      // Never leave a CTA with copies in flight: on an abort, wait (bounded) for the
      // last load issued to each stage.
      if (*s_abort) {
        volatile int local_abort = 0;
        for (int kb = max(0, issued - STAGES); kb < issued; ++kb)
          ptx::mbar_wait_bounded(&full[kb % STAGES], (kb / STAGES) & 1, &local_abort, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16_f32(kBM, BN);
      bool committed_any = false;
      int kb = 0;
      for (; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!ptx::mbar_wait_bounded(&full[s], ph, s_abort, kWaitLimitNs)) break;
        if (!ptx::mbar_wait_bounded(&afull[s], ph, s_abort, kWaitLimitNs)) break;
        ptx::tc_fence_after();
        const uint64_t bdesc = ptx::smem_desc_k_sw128(act_s(s));
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint32_t a_tmem = tmem + C::A0 + 32 * s + 8 * kk;
          ptx::mma_f16_ts(tmem /*D at column 0*/, a_tmem, bdesc + 2 * kk, idesc, (kb | kk) != 0);
        }
        ptx::tc_commit(&empty[s]);
        committed_any = true;
      }
      ptx::tc_commit(accf);  // arrives once every MMA above has completed
      if (*s_abort && committed_any) {
        volatile int local_abort = 0;
        ptx::mbar_wait_bounded(accf, 0, &local_abort, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ decode warps
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;       // weight row of the tile == TMEM lane
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const bool row_valid = row < 64 || halfB;
    const int scale_off = (row < 64) ? row : 128 + (row - 64);   // [half][c][64]
    constexpr int scale_kstride = 64;
    bool range_bad = false;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!ptx::mbar_wait_bounded(&full[s], ph, s_abort, kWaitLimitNs)) break;
      const uint8_t* cbase = code_s(s) + row * 32;
      const int sw = (row >> 2) & 1;      // 32-byte swizzle: 16-byte chunk index ^= row bit 2
      const uint4 c0 = *reinterpret_cast<const uint4*>(cbase + ((0 ^ sw) << 4));
      const uint4 c1 = *reinterpret_cast<const uint4*>(cbase + ((1 ^ sw) << 4));
      const int sb0 = scale_s(s)[scale_off];
      const int sb1 = scale_s(s)[scale_off + scale_kstride];
      uint32_t m0 = f16_pow2_bits(sb0 - 127), m1 = f16_pow2_bits(sb1 - 127);
      if (row_valid && (m0 == 0u || m1 == 0u)) range_bad = true;
      m0 |= m0 << 16;
      m1 |= m1 << 16;
      uint32_t r[32];
      const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t o0, o1, o2, o3;
        ptx::e2m1x8_to_f16x8(cw[i], o0, o1, o2, o3);
        const uint32_t m = row_valid ? ((i < 4) ? m0 : m1) : 0u;   // rows past the matrix: zeros
        r[4 * i + 0] = ptx::hmul2_u32(o0, m);
        r[4 * i + 1] = ptx::hmul2_u32(o1, m);
        r[4 * i + 2] = ptx::hmul2_u32(o2, m);
        r[4 * i + 3] = ptx::hmul2_u32(o3, m);
      }
      ptx::tmem_st32(tmem + lane_addr + C::A0 + 32 * s, r);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&afull[s]);
    }
    if (range_bad) set_status(p.status, MOE_ERR_RANGE);

    // ------------------------------------------------------------------ epilogue
    if (!*s_abort) ptx::mbar_wait_bounded(accf, 0, s_abort, kWaitLimitNs);
    // Agree on the outcome before any named barrier: after this barrier nothing can
    // raise the abort flag any more (producer and MMA issuer are done), so every
    // epilogue thread reads the same value.
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const bool ok = !*s_abort;
    ptx::tc_fence_after();
    if (ok) {
      const int et = threadIdx.x - 64;  // 0..127 over the four epilogue warps
      if (MODE == MODE_GATE_UP) {
        // Per 32-token chunk the gate thread of column j (lane row j < 64) and the up
        // thread of the same column (row j + 64) trade halves: the gate side finishes
        // tokens 0..15 of the chunk, the up side tokens 16..31.
        float* s_x = reinterpret_cast<float*>(smem);                       // [32][64] exchange
        uint16_t* s_h = reinterpret_cast<uint16_t*>(smem + 32 * 64 * 4);  // [BN][64]
        const float L = p.limit;
        const bool gate_side = row < 64;
        const int j = gate_side ? row : row - 64;
        constexpr int CW = BN < 32 ? BN : 32;   // accumulator columns per chunk
        constexpr int HW = CW / 2;              // tokens each side finishes
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(tmem + lane_addr + c0, v);
          ptx::tmem_wait_ld();
          // gate side publishes its g for the upper half, up side its u for the lower half
#pragma unroll
          for (int c = 0; c < HW; ++c) {
            const int cc = gate_side ? HW + c : c;
            s_x[cc * 64 + j] = __uint_as_float(v[cc]);
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
          for (int c = 0; c < HW; ++c) {
            const int cc = gate_side ? c : HW + c;
            const float mine = __uint_as_float(v[cc]);
            const float other = s_x[cc * 64 + j];
            const float g = fminf(gate_side ? mine : other, L);
            const float u = fminf(fmaxf(gate_side ? other : mine, -L), L);
            const float hval = g * __frcp_rn(1.0f + __expf(-g)) * u;   // silu(g) * u
            uint32_t b = __float_as_uint(hval);
            b = (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;       // round to bf16
            s_h[(c0 + cc) * 64 + j] = __half_as_ushort(__float2half_rn(__uint_as_float(b)));
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        // rows of h: token t -> 64 f16 = 8 x 16 B
        for (int i = et; i < tl.rows * 8; i += 128) {
          const int t = i >> 3, c = i & 7;
          const uint4 val = *reinterpret_cast<const uint4*>(s_h + t * 64 + c * 8);
          *reinterpret_cast<uint4*>(p.h_out + (int64_t)(tl.row0 + t) * p.I + row_tile0 + c * 8) = val;
        }
      } else {
        float* s_y = reinterpret_cast<float*>(smem);  // [BN][128]
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(tmem + lane_addr + c0, v);
          ptx::tmem_wait_ld();
          constexpr int CW = BN < 32 ? BN : 32;
#pragma unroll
          for (int c = 0; c < CW; ++c) s_y[(c0 + c) * 128 + row] = __uint_as_float(v[c]);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int ncol = min(128, p.d - row_tile0);
        const int n4 = ncol / 4;
        for (int i = et; i < tl.rows * 32; i += 128) {
          const int t = i >> 5, c4 = i & 31;
          if (c4 >= n4) continue;
          const float wgt = p.w_sorted[tl.row0 + t];
          float4 val = *reinterpret_cast<const float4*>(s_y + t * 128 + c4 * 4);
          val.x *= wgt;
          val.y *= wgt;
          val.z *= wgt;
          val.w *= wgt;
          *reinterpret_cast<float4*>(p.ys_out + (int64_t)(tl.row0 + t) * p.d + row_tile0 + c4 * 4) = val;
        }
      }
    }
  }

  __syncthreads();
  if (*s_abort && threadIdx.x == 0) set_status(p.status, MOE_ERR_TIMEOUT);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  return fn(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int BN, int STAGES>
int launch_one(const FwdArgs& a) {
  using C = Cfg<BN, STAGES>;
  const int P = a.T * a.k;
  const int K = (MODE == MODE_GATE_UP) ? a.d : a.I;
  const int R = (MODE == MODE_GATE_UP) ? 2 * a.I : a.d;  // weight rows per expert
  const uint8_t* codes = (MODE == MODE_GATE_UP) ? a.w1c : a.w2c;
  const uint8_t* scales = (MODE == MODE_GATE_UP) ? a.w1s : a.w2s;
  const uint16_t* act = (MODE == MODE_GATE_UP) ? a.ws.xs : a.ws.h;

  CUtensorMap m_act;
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)P};
    const uint64_t str[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {kBK, BN};
    if (!make_map(&m_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, act, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return -1;
  }
  TcParams prm;
  prm.tiles = a.ws.tiles;
  prm.ntiles = a.ws.ntiles;
  prm.codes = codes;
  prm.scales = scales;
  prm.N = R;
  prm.w_sorted = a.ws.w_sorted;
  prm.h_out = a.ws.h;
  prm.ys_out = a.ws.ys;
  prm.status = a.ws.status;
  prm.K = K;
  prm.I = a.I;
  prm.d = a.d;
  prm.limit = a.limit;

  auto kern = tc_expert_kernel<MODE, BN, STAGES>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return -1;
  const int max_tiles = (P + BN - 1) / BN + a.E;
  const int row_tiles = (MODE == MODE_GATE_UP) ? a.I / 64 : (a.d + kBM - 1) / kBM;
  ev_before(a);
  kern<<<dim3(max_tiles, row_tiles), kThreads, C::SMEM_BYTES, a.stream>>>(m_act, prm);
  ev_after(a);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

constexpr int kGemvBN = 16, kGemvStages = 6;
constexpr int kGemmBN = 128, kGemmStages = 4;

}  // namespace

int tc_tile_tokens(int path) { return path == MOE_PATH_GEMV ? kGemvBN : kGemmBN; }

int launch_experts_tc(const FwdArgs& a, int tile_tokens) {
  int n1, n2;
  if (tile_tokens == kGemvBN) {
    n1 = launch_one<MODE_GATE_UP, kGemvBN, kGemvStages>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, kGemvBN, kGemvStages>(a);
  } else {
    n1 = launch_one<MODE_GATE_UP, kGemmBN, kGemmStages>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, kGemmBN, kGemmStages>(a);
  }
  if (n2 < 0) return -1;
  return n1 + n2;
}

}  // namespace moe
