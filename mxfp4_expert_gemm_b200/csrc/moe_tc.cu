// tcgen05 grouped expert GEMMs: gate_up with the clamped-SwiGLU epilogue, and down
// with the routing-weight epilogue.
//
// Layer definition: the SwiGLU expert of "From GPT-2 to gpt-oss" (新智元
// translation), sec. 3 (three linears, silu(z) = z * sigmoid(z)), with
// swiglu_limit 7 from the llm-atlas GPT-OSS 20B config table; MXFP4 weights per the
// ewbang.com GPT-OSS article, section 量化 (E2M1 values, one E8M0 scale per 32).
//
// Persistent kernel, CPS CTAs per SM.  A work item is a 128 (weight rows) x BN (tokens
// of one expert) output tile over the whole reduction axis; CTA b takes items b,
// b + grid, ...  A pipeline stage covers KS of the reduction axis (KS/64 chunks of 64;
// the last stage of a row may hold fewer).  The weights are the MMA's A operand and
// live in TMEM:
//   warp 0        producer: per stage one 3D TMA load of the activation tile
//                 [KS/64][BN][64] (128B swizzle) and one bulk copy per 64-row weight half
//                 for the codes (KS/64 consecutive 2 KB blocks) and one for the scales;
//                 lane 0 issues the TMA, lanes 1..4 the bulk copies;
//   warp 1        TMEM allocation and the MMA issuer (one thread);
//   decode warps  DG groups of 4 warps; group q decodes the stages with
//                 stage % DG == q.  Each thread owns one weight row (= its TMEM lane),
//                 turns 32 code bytes per chunk into 64 f16 values (E2M1 -> f16
//                 convert, times the exact power-of-two scale) and stores them to the
//                 stage's TMEM A slot;
//   epilogue      4 warps read the fp32 accumulator (double-buffered in TMEM, so the
//                 epilogue of one item overlaps the main loop of the next) and write
//                 h (gate_up) or the routing-weighted expert output (down).
// The decoded weights never touch shared memory: the tensor core's only shared-memory
// operand is the activation tile.
//
// Gate_up tiles hold 64 gate rows (TMEM lanes 0..63) and the 64 matching up rows
// (lanes 64..127), so g and u of one output column meet in the epilogue.
//
// Every wait is bounded (kWaitLimitNs).  When one gives up, the CTA raises its abort
// flag, every role leaves its loop, in-flight copies and MMAs are drained (bounded),
// TMEM is freed and MOE_ERR_TIMEOUT is recorded.
#include <cuda.h>
#include <cuda_fp16.h>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;                          // weight rows per tile (TMEM lanes)
constexpr int kCK = 64;                           // K per chunk (one weight block, one swizzle row)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: a stuck pipeline, not a slow one

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct TcParams {
  const Tile* tiles;
  const int32_t* ntiles;
  const uint8_t* codes;   // MXFP4 codes of W1 or W2 (library block layout)
  const uint8_t* scales;
  int32_t N;              // weight rows per expert (2I or d)
  const float* w_sorted;
  uint16_t* h_out;        // gate_up: [P][I] f16
  float* ys_out;          // down:    [P][d] f32
  int32_t* status;
  int32_t K;              // reduction length (d for gate_up, I for down)
  int32_t nchunks;        // K / 64
  int32_t act_box_bytes;  // bytes one activation TMA box brings (min(KS, K)/64 chunks)
  int32_t I, d;
  int32_t n_rt;           // row tiles per token tile
  float limit;
  int32_t inject_timeout; // test hook: CTA 0 withholds its first decode arrival
  // fused combine (down): y = bf16(x + sum_j ys[inv[t*k + j]]) by the last writer of a
  // (token, 128-column) block
  int32_t fuse_combine;
  int32_t k;
  const int32_t* perm;
  const int32_t* inv;
  const uint16_t* x;
  uint16_t* y;
  int32_t* arrivals;
};

template <int BN, int KS, int S, int SA, int DG, int CPS>
struct Cfg {
  static constexpr int NC = KS / kCK;                          // chunks per stage
  static constexpr int ACT_CHUNK = BN * 128;                   // one 64-wide activation chunk
  static constexpr int ACT_BYTES = NC * ACT_CHUNK;
  static constexpr int CODE_HALF = NC * kBlkCodeBytes;         // one 64-row half, NC blocks
  static constexpr int SCALE_HALF = NC * kBlkScaleBytes;
  static constexpr int CODE_OFF = ACT_BYTES;
  static constexpr int SCALE_OFF = ACT_BYTES + 2 * CODE_HALF;
  static constexpr int STAGE_BYTES = ((ACT_BYTES + 2 * CODE_HALF + 2 * SCALE_HALF + 1023) / 1024) * 1024;
  static constexpr int ACC_COLS = BN < 32 ? 32 : BN;           // one accumulator buffer
  static constexpr int A0 = 2 * ACC_COLS;                      // first column of the A slots
  static constexpr int SLOT_COLS = KS / 2;                     // f16 pairs per row per stage
  static constexpr int COLS_NEEDED = A0 + SLOT_COLS * SA;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 64 ? 64 : COLS_NEEDED <= 128 ? 128
                                   : COLS_NEEDED <= 256 ? 256 : 512;
  static constexpr int EPI_GU = 32 * 64 * 4 + BN * 64 * 2;     // exchange + h staging
  static constexpr int EPI_DN = 32 * 128 * 4 + 32 * 4;         // one 32-token chunk + token ids
  static constexpr int EPI_BYTES = EPI_GU > EPI_DN ? EPI_GU : EPI_DN;
  static constexpr int BAR_BYTES = 8 * (2 * S + 2 * SA + 4 + 1) + 16;
  static constexpr int SMEM_BYTES = S * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024 /*align slack*/;
  static constexpr int WARPS = 2 + 4 * DG + 4;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int EPI_WARP0 = 2 + 4 * DG;
  static_assert(KS % kCK == 0 && NC >= 1, "stage = whole chunks");
  static_assert(TMEM_COLS * CPS <= 512, "TMEM budget of CPS co-resident CTAs");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M = 128");
  static_assert(SMEM_BYTES * CPS <= 226 * 1024, "shared memory budget of CPS co-resident CTAs");
};

// f16 bit pattern of 2^e, or 0 when E2M1 * 2^e is not exact in f16 (e outside [-23, 13]).
__device__ __forceinline__ uint32_t f16_pow2_bits(int e) {
  if (e > 13 || e < -23) return 0u;
  if (e >= -14) return (uint32_t)(e + 15) << 10;   // normal
  return 1u << (e + 24);                            // subnormal 2^-15 .. 2^-23
}

struct Item {
  Tile tl;
  int rt;
  int row_tile0;
  int rbA, rbB;
  bool halfB;
};

template <int MODE>
__device__ __forceinline__ Item item_of(const TcParams& p, int i) {
  Item it;
  const int tt = i / p.n_rt, rt = i - tt * p.n_rt;
  it.tl = p.tiles[tt];
  it.rt = rt;
  it.row_tile0 = (MODE == MODE_GATE_UP) ? rt * 64 : rt * kBM;
  it.rbA = it.row_tile0 / kBlkRows;
  // gate_up pairs gate rows j0.. with up rows I+j0..; down takes rows m0.. and m0+64..
  it.rbB = (MODE == MODE_GATE_UP) ? (p.I + it.row_tile0) / kBlkRows : it.rbA + 1;
  it.halfB = it.rbB < p.N / kBlkRows;
  return it;
}

template <int MODE, int BN, int KS, int S, int SA, int DG, int CPS>
__global__ void __launch_bounds__(Cfg<BN, KS, S, SA, DG, CPS>::THREADS, CPS)
    tc_expert_kernel(const __grid_constant__ CUtensorMap tm_act, const TcParams p) {
  using C = Cfg<BN, KS, S, SA, DG, CPS>;
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + S * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + C::EPI_BYTES);
  uint64_t* sfree = full + S;       // SMEM slot consumed (MMA done)
  uint64_t* afull = sfree + S;      // TMEM A slot written (decode done)
  uint64_t* afree = afull + SA;     // TMEM A slot consumed (MMA done)
  uint64_t* accf = afree + SA;      // [2] accumulator ready
  uint64_t* acce = accf + 2;        // [2] accumulator drained by the epilogue
  uint64_t* drain = acce + 2;       // final MMA drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.nchunks + C::NC - 1) / C::NC;   // stages per item

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&sfree[s], 1);
    }
    for (int a = 0; a < SA; ++a) {
      ptx::mbar_init(&afull[a], 128);
      ptx::mbar_init(&afree[a], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&accf[b], 1);
      ptx::mbar_init(&acce[b], 128);
    }
    ptx::mbar_init(drain, 1);
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
  // Everything above overlaps the previous kernel; the work list is its output.
  pdl_wait();
  const int n_items = *p.ntiles * p.n_rt;

  auto act_s = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto code_s = [&](int s) { return smem + s * C::STAGE_BYTES + C::CODE_OFF; };
  auto scale_s = [&](int s) { return smem + s * C::STAGE_BYTES + C::SCALE_OFF; };
  auto chunks_of = [&](int kb) { return min(C::NC, p.nchunks - kb * C::NC); };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // Lane 0 owns the ring; lanes 1..4 issue the bulk copies of a stage in one warp
    // instruction (codes A, codes B, scales A, scales B).
    int64_t g = 0;  // global stage counter of this CTA
    bool stop = false;
    for (int i = blockIdx.x; i < n_items && !stop; i += gridDim.x) {
      const Item it = item_of<MODE>(p, i);
      const int halves = it.halfB ? 2 : 1;
      for (int kb = 0; kb < nk; ++kb, ++g) {
        const int s = (int)(g % S);
        const int nck = chunks_of(kb);
        bool ok = true;
        if (lane == 0) {
          if (g >= S) ok = ptx::mbar_wait_bounded(&sfree[s], (uint32_t)((g / S) - 1) & 1, s_abort, kWaitLimitNs);
          if (ok) {
            const uint32_t tx = p.act_box_bytes + halves * nck * (kBlkCodeBytes + kBlkScaleBytes);
            ptx::mbar_arrive_expect_tx(&full[s], tx);
            ptx::tma_load_3d(act_s(s), &tm_act, 0, it.tl.row0, kb * C::NC, &full[s]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) {
          stop = true;
          break;
        }
        if (lane >= 1 && lane <= 4) {
          const int half = (lane - 1) & 1;     // lanes 1, 3: half A; lanes 2, 4: half B
          const bool scales = lane >= 3;
          if (half == 0 || it.halfB) {
            const int64_t blk = mx_block_index(it.tl.e, half ? it.rbB : it.rbA, (int64_t)kb * C::NC, p.N, p.K);
            if (scales)
              ptx::bulk_load(scale_s(s) + half * C::SCALE_HALF, p.scales + blk * kBlkScaleBytes,
                             nck * kBlkScaleBytes, &full[s]);
            else
              ptx::bulk_load(code_s(s) + half * C::CODE_HALF, p.codes + blk * kBlkCodeBytes, nck * kBlkCodeBytes,
                             &full[s]);
          }
        }
        __syncwarp();
      }
    }
    // Never leave copies in flight when the CTA exits (consumers may have aborted before
    // waiting for them): wait, bounded, for the last fill of every slot.  On the normal
    // path these have all landed already.
    if (lane == 0) {
      volatile int local_abort = 0;
      for (int64_t q = (g > S ? g - S : 0); q < g; ++q)
        ptx::mbar_wait_bounded(&full[q % S], (uint32_t)(q / S) & 1, &local_abort, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16_f32(kBM, BN);
      int64_t g = 0;
      int li = 0;
      bool stop = false;
      for (int i = blockIdx.x; i < n_items && !stop; i += gridDim.x, ++li) {
        const int b = li & 1;
        if (li >= 2 && !ptx::mbar_wait_bounded(&acce[b], (uint32_t)((li >> 1) - 1) & 1, s_abort, kWaitLimitNs))
          break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + b * C::ACC_COLS;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % S), a = (int)(g % SA);
          if (!ptx::mbar_wait_bounded(&full[s], (uint32_t)(g / S) & 1, s_abort, kWaitLimitNs) ||
              !ptx::mbar_wait_bounded(&afull[a], (uint32_t)(g / SA) & 1, s_abort, kWaitLimitNs)) {
            stop = true;
            break;
          }
          ptx::tc_fence_after();
          const int nck = chunks_of(kb);
          for (int j = 0; j < nck; ++j) {
            const uint64_t bdesc = ptx::smem_desc_k_sw128(act_s(s) + j * C::ACT_CHUNK);
            const uint32_t a_tmem = tmem + C::A0 + C::SLOT_COLS * a + 32 * j;
#pragma unroll
            for (int kk = 0; kk < kCK / 16; ++kk)
              ptx::mma_f16_ts(d_tmem, a_tmem + 8 * kk, bdesc + 2 * kk, idesc, (kb | j | kk) != 0);
          }
          ptx::tc_commit(&sfree[s]);
          ptx::tc_commit(&afree[a]);
        }
        if (!stop) ptx::tc_commit(&accf[b]);
      }
      // Every MMA issued above completes before the drain barrier fires.
      ptx::tc_commit(drain);
      volatile int local_abort = 0;
      ptx::mbar_wait_bounded(drain, 0, &local_abort, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp < C::EPI_WARP0) {
    // ------------------------------------------------------------------ decode warps
    // Per chunk: convert into one of two register buffers and issue its TMEM store; the
    // stores of a stage complete (wait::st) together before the stage is handed to the
    // MMA issuer.  Alternating buffers keep a register that a store may still read from
    // being overwritten.
    const int grp = (warp - 2) >> 2;     // decode group: stages with g % DG == grp
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;       // weight row of the tile == TMEM lane
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const int half = row >> 6, rr = row & 63;
    const int code_off = half * C::CODE_HALF + rr * 32;
    const int scale_off = half * C::SCALE_HALF + rr;
    const int sw = (rr >> 2) & 1;       // chunk swizzle of the block layout
    bool range_bad = false, stop = false;
    uint32_t r0[32], r1[32];
    auto convert = [&](uint32_t (&r)[32], int s, int j, bool row_valid) {
      const uint8_t* cbase = code_s(s) + code_off + j * kBlkCodeBytes;
      const uint4 c0 = *reinterpret_cast<const uint4*>(cbase + ((0 ^ sw) << 4));
      const uint4 c1 = *reinterpret_cast<const uint4*>(cbase + ((1 ^ sw) << 4));
      const uint8_t* sbase = scale_s(s) + scale_off + j * kBlkScaleBytes;
      uint32_t m0 = f16_pow2_bits((int)sbase[0] - 127), m1 = f16_pow2_bits((int)sbase[64] - 127);
      if (row_valid && (m0 == 0u || m1 == 0u)) range_bad = true;
      if (!row_valid) m0 = m1 = 0u;  // rows past the matrix: zeros
      m0 |= m0 << 16;
      m1 |= m1 << 16;
      const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        uint32_t o0, o1, o2, o3;
        ptx::e2m1x8_to_f16x8(cw[jj], o0, o1, o2, o3);
        const uint32_t m = (jj < 4) ? m0 : m1;
        r[4 * jj + 0] = ptx::hmul2_u32(o0, m);
        r[4 * jj + 1] = ptx::hmul2_u32(o1, m);
        r[4 * jj + 2] = ptx::hmul2_u32(o2, m);
        r[4 * jj + 3] = ptx::hmul2_u32(o3, m);
      }
    };
    int64_t g = 0;
    for (int i = blockIdx.x; i < n_items && !stop; i += gridDim.x) {
      const Item it = item_of<MODE>(p, i);
      const bool row_valid = half == 0 || it.halfB;
      for (int kb = 0; kb < nk; ++kb, ++g) {
        if ((int)(g % DG) != grp) continue;
        const int s = (int)(g % S), a = (int)(g % SA);
        if (!ptx::mbar_wait_bounded(&full[s], (uint32_t)(g / S) & 1, s_abort, kWaitLimitNs) ||
            (g >= SA &&
             !ptx::mbar_wait_bounded(&afree[a], (uint32_t)((g / SA) - 1) & 1, s_abort, kWaitLimitNs))) {
          stop = true;
          break;
        }
        const int nck = chunks_of(kb);
        const uint32_t slot = tmem + lane_addr + C::A0 + C::SLOT_COLS * a;
#pragma unroll
        for (int j = 0; j < C::NC; ++j) {
          if (j < nck) {
            if (j & 1) {
              convert(r1, s, j, row_valid);
              ptx::tmem_st32(slot + 32 * j, r1);
            } else {
              convert(r0, s, j, row_valid);
              ptx::tmem_st32(slot + 32 * j, r0);
            }
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        if (!(p.inject_timeout && blockIdx.x == 0 && g == 0)) ptx::mbar_arrive(&afull[a]);
      }
    }
    if (range_bad) set_status(p.status, MOE_ERR_RANGE);
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const int et = threadIdx.x - 32 * C::EPI_WARP0;  // 0..127
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    int li = 0;
    for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++li) {
      const int b = li & 1;
      const bool ready = !*s_abort && ptx::mbar_wait_bounded(&accf[b], (uint32_t)(li >> 1) & 1, s_abort,
                                                             kWaitLimitNs);
      // The four epilogue warps take the same branch (the abort flag may be raised by
      // another role at any time; the barrier reduction freezes one answer for all).
      if (ptx::bar_or<1, 128>(!ready)) break;
      ptx::tc_fence_after();
      const Item it = item_of<MODE>(p, i);
      const uint32_t acc = tmem + lane_addr + b * C::ACC_COLS;
      if (MODE == MODE_GATE_UP) {
        // Per 32-token chunk the gate thread of column j (row j < 64) and the up thread of
        // the same column (row j + 64) trade halves: the gate side finishes tokens 0..15
        // of the chunk, the up side tokens 16..31.
        float* s_x = reinterpret_cast<float*>(epi);                       // [32][64] exchange
        uint16_t* s_h = reinterpret_cast<uint16_t*>(epi + 32 * 64 * 4);  // [BN][64]
        const float L = p.limit;
        const bool gate_side = row < 64;
        const int j = gate_side ? row : row - 64;
        constexpr int CW = BN < 32 ? BN : 32;
        constexpr int HW = CW / 2;
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(acc + c0, v);
          ptx::tmem_wait_ld();
          // (register indices stay compile-time constants: select values, not indices)
#pragma unroll
          for (int c = 0; c < HW; ++c) {
            const int cc = gate_side ? HW + c : c;
            s_x[cc * 64 + j] = __uint_as_float(gate_side ? v[HW + c] : v[c]);
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
          for (int c = 0; c < HW; ++c) {
            const int cc = gate_side ? c : HW + c;
            const float mine = __uint_as_float(gate_side ? v[c] : v[HW + c]);
            const float other = s_x[cc * 64 + j];
            const float gv = fminf(gate_side ? mine : other, L);
            const float uv = fminf(fmaxf(gate_side ? other : mine, -L), L);
            const float hval = gv * __frcp_rn(1.0f + __expf(-gv)) * uv;   // silu(g) * u
            uint32_t bits = __float_as_uint(hval);
            bits = (bits + 0x7FFFu + ((bits >> 16) & 1u)) & 0xFFFF0000u;    // round to bf16
            s_h[(c0 + cc) * 64 + j] = __half_as_ushort(__float2half_rn(__uint_as_float(bits)));
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        // The accumulator is no longer needed: hand it back to the MMA issuer.
        ptx::tc_fence_before();
        ptx::mbar_arrive(&acce[b]);
        // rows of h: token t -> 64 f16 = 8 x 16 B
        for (int idx = et; idx < it.tl.rows * 8; idx += 128) {
          const int t = idx >> 3, c = idx & 7;
          const uint4 val = *reinterpret_cast<const uint4*>(s_h + t * 64 + c * 8);
          *reinterpret_cast<uint4*>(p.h_out + (int64_t)(it.tl.row0 + t) * p.I + it.row_tile0 + c * 8) = val;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");  // s_h is reused by the next item
      } else {
        float* s_y = reinterpret_cast<float*>(epi);  // [32 tokens][128]
        const int ncol = min(128, p.d - it.row_tile0);
        const int n4 = ncol / 4;
        constexpr int CW = BN < 32 ? BN : 32;
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(acc + c0, v);
          ptx::tmem_wait_ld();
          if (c0 + 32 >= BN) {  // last chunk read: the accumulator goes back to the MMA issuer
            ptx::tc_fence_before();
            ptx::mbar_arrive(&acce[b]);
          }
#pragma unroll
          for (int c = 0; c < CW; ++c) s_y[c * 128 + row] = __uint_as_float(v[c]);
          asm volatile("bar.sync 1, 128;" ::: "memory");
          const int nt = min(CW, it.tl.rows - c0);
          for (int idx = et; idx < nt * 32; idx += 128) {
            const int t = idx >> 5, c4 = idx & 31;
            if (c4 >= n4) continue;
            const int prow = it.tl.row0 + c0 + t;
            const float wgt = p.w_sorted[prow];
            float4 val = *reinterpret_cast<const float4*>(s_y + t * 128 + c4 * 4);
            val.x *= wgt;
            val.y *= wgt;
            val.z *= wgt;
            val.w *= wgt;
            *reinterpret_cast<float4*>(p.ys_out + (int64_t)prow * p.d + it.row_tile0 + c4 * 4) = val;
          }
          if (p.fuse_combine) {
            // Publish this chunk's outputs, count them per (token, column block); the writer of
            // a token's k-th contribution adds the k outputs in slot order plus the residual.
            int* s_tok = reinterpret_cast<int*>(s_y + 32 * 128) - 0;  // reuse past the staging rows
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (et < nt) {
              const int tok = p.perm[it.tl.row0 + c0 + et] / p.k;
              const int prev = atomicAdd(p.arrivals + (int64_t)tok * p.n_rt + it.rt, 1);
              s_tok[et] = (prev == p.k - 1) ? tok : -1;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            __threadfence();
            for (int t = 0; t < nt; ++t) {
              const int tok = s_tok[t];
              if (tok < 0) continue;
              for (int col = et; col < ncol; col += 128) {
                const int64_t gc = it.row_tile0 + col;
                float acc = __uint_as_float((uint32_t)p.x[(int64_t)tok * p.d + gc] << 16);
                for (int j = 0; j < p.k; ++j) {
                  const int srow = p.inv[(int64_t)tok * p.k + j];
                  acc += __ldcg(p.ys_out + (int64_t)srow * p.d + gc);
                }
                uint32_t b = __float_as_uint(acc);
                b = (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;   // round to bf16
                p.y[(int64_t)tok * p.d + gc] = (uint16_t)b;
              }
            }
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
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

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

template <int MODE, int BN, int KS, int S, int SA, int DG, int CPS>
int launch_one(const FwdArgs& a) {
  using C = Cfg<BN, KS, S, SA, DG, CPS>;
  const int P = a.T * a.k;
  const int K = (MODE == MODE_GATE_UP) ? a.d : a.I;
  const int R = (MODE == MODE_GATE_UP) ? 2 * a.I : a.d;  // weight rows per expert
  const uint8_t* codes = (MODE == MODE_GATE_UP) ? a.w1c : a.w2c;
  const uint8_t* scales = (MODE == MODE_GATE_UP) ? a.w1s : a.w2s;
  const uint16_t* act = (MODE == MODE_GATE_UP) ? a.ws.xs : a.ws.h;

  // Activations [P][K] f16 viewed as [K/64 chunks][P rows][64]: one box brings the
  // stage's KS/64 chunks of BN rows, each chunk a 128B-swizzled [BN][64] tile.
  CUtensorMap m_act;
  {
    const uint64_t dims[3] = {(uint64_t)kCK, (uint64_t)P, (uint64_t)K / kCK};
    const uint64_t str[2] = {(uint64_t)K * 2, (uint64_t)kCK * 2};
    const uint32_t box[3] = {kCK, BN, (uint32_t)std::min(C::NC, K / kCK)};
    if (!make_map(&m_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, act, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
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
  prm.nchunks = K / kCK;
  prm.act_box_bytes = std::min(C::NC, K / kCK) * C::ACT_CHUNK;
  prm.I = a.I;
  prm.d = a.d;
  prm.n_rt = (MODE == MODE_GATE_UP) ? a.I / 64 : (a.d + kBM - 1) / kBM;
  prm.limit = a.limit;
  prm.inject_timeout = (MODE == MODE_GATE_UP) ? a.inject_timeout : 0;
  prm.fuse_combine = (MODE == MODE_DOWN) ? a.fuse_combine : 0;
  prm.k = a.k;
  prm.perm = a.ws.perm;
  prm.inv = a.ws.inv;
  prm.x = a.x;
  prm.y = a.y;
  prm.arrivals = a.ws.arrivals;

  auto kern = tc_expert_kernel<MODE, BN, KS, S, SA, DG, CPS>;
  static std::atomic<uint64_t> attr_done{0};   // per-device "attribute set" bits
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return -1;
    attr_done.fetch_or(bit, std::memory_order_release);
  }
  const int64_t max_items = (int64_t)((P + BN - 1) / BN + a.E) * prm.n_rt;
  const int grid = (int)std::min<int64_t>(max_items, (int64_t)sm_count() * CPS);
  ev_before(a);
  if (launch_kernel(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, a.stream, a.pdl != 0, m_act, prm) !=
      cudaSuccess)
    return -1;
  ev_after(a);
  return 1;
}

// Pipeline shapes (compile-time; overridable with -D for tuning builds).
// Small batches (few tokens per expert): 16-token tiles, 192-wide stages, two
// independent pipelines (CTAs) per SM.
#ifndef MOE_GEMV_KS
#define MOE_GEMV_KS 192
#endif
#ifndef MOE_GEMV_S
#define MOE_GEMV_S 5
#endif
#ifndef MOE_GEMV_SA
#define MOE_GEMV_SA 2
#endif
#ifndef MOE_GEMV_DG
#define MOE_GEMV_DG 1
#endif
#ifndef MOE_GEMV_CPS
#define MOE_GEMV_CPS 2
#endif
// Large batches: 128-token tiles, 192-wide stages.
#ifndef MOE_GEMM_KS
#define MOE_GEMM_KS 192
#endif
#ifndef MOE_GEMM_S
#define MOE_GEMM_S 3
#endif
#ifndef MOE_GEMM_SA
#define MOE_GEMM_SA 2
#endif
#ifndef MOE_GEMM_DG
#define MOE_GEMM_DG 2
#endif
#ifndef MOE_GEMM_CPS
#define MOE_GEMM_CPS 1
#endif
constexpr int kGemvBN = 16, kGemvKS = MOE_GEMV_KS, kGemvS = MOE_GEMV_S, kGemvSA = MOE_GEMV_SA,
              kGemvDG = MOE_GEMV_DG, kGemvCPS = MOE_GEMV_CPS;
constexpr int kGemmBN = 128, kGemmKS = MOE_GEMM_KS, kGemmS = MOE_GEMM_S, kGemmSA = MOE_GEMM_SA,
              kGemmDG = MOE_GEMM_DG, kGemmCPS = MOE_GEMM_CPS;

}  // namespace

int tc_tile_tokens(int path) { return path == MOE_PATH_GEMV ? kGemvBN : kGemmBN; }

int launch_experts_tc(const FwdArgs& a, int tile_tokens) {
  int n1, n2;
  if (tile_tokens == kGemvBN) {
    n1 = launch_one<MODE_GATE_UP, kGemvBN, kGemvKS, kGemvS, kGemvSA, kGemvDG, kGemvCPS>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, kGemvBN, kGemvKS, kGemvS, kGemvSA, kGemvDG, kGemvCPS>(a);
  } else {
    n1 = launch_one<MODE_GATE_UP, kGemmBN, kGemmKS, kGemmS, kGemmSA, kGemmDG, kGemmCPS>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, kGemmBN, kGemmKS, kGemmS, kGemmSA, kGemmDG, kGemmCPS>(a);
  }
  if (n2 < 0) return -1;
  return n1 + n2;
}

}  // namespace moe
