// Block-scaled tcgen05 grouped expert GEMMs: gate_up with the clamped-SwiGLU epilogue,
// and down with the routing-weight epilogue.
//
// Layer definition: the SwiGLU expert of "From GPT-2 to gpt-oss" (新智元
// translation), sec. 3 (three linears, silu(z) = z * sigmoid(z)), with
// swiglu_limit 7 from the llm-atlas GPT-OSS 20B config table; MXFP4 weights per the
// ewbang.com GPT-OSS article, section 量化 (E2M1 values, one E8M0 scale per 32).
//
// The tensor cores read the MXFP4 weights as stored: tcgen05.mma kind::mxf8f6f4 with an
// E2M1 A operand (the weights, 128 rows per tile) scaled by its E8M0 block scales, and an
// E4M3 B operand (the activations) scaled by theirs; fp32 accumulation in TMEM.  With bf16
// activations each activation vector is two B columns, its hi and lo E4M3 terms (see
// e4m3_split), so a tile of BN tokens is an MMA of N = 2*BN and the epilogue adds column
// pairs (TERMS = 2); with MXFP8 activations a token is one column (TERMS = 1).
//
// Persistent kernel, CPS CTAs per SM.  A work item is 128 weight rows x one token tile
// over the whole reduction axis (or a split of it); CTA b takes items b, b + grid, ...
// With CG = 2 (large batches) two CTAs of a cluster share each MMA of M = 256: a pair
// takes two consecutive row tiles of an item, each CTA holding its weight rows and half
// of the token tile's activation rows (the CG == 2 branches below).  A pipeline stage covers NP
// chunks of 128 along the reduction axis:
//   warps 0..  producers: per stage one TMA load of the weight codes (NP consecutive
//              8 KB tile blocks; E2M1, unpacked by the copy to one byte per code in
//              shared memory, 128B swizzle), one bulk copy of the token tile's packed
//              activation blocks (TERMS*BN E4M3 rows per chunk, already in the swizzled order,
//              followed by their scale factors) and one bulk copy of the weight scale
//              factors (stored in the tensor cores' scale-factor layout); pairs load the
//              same by tile copies that complete on the leader's barrier;
//   warp NPW   TMEM allocation and the MMA issuer (one elected thread): per stage it
//              copies the scale factors into TMEM (tcgen05.cp) and issues one block-scaled
//              MMA per 32-wide block of the reduction axis (pairs: the leader's only);
//   then       epilogue, EG warpgroups taking alternate 32-column reads: read the fp32
//              accumulator (double-buffered in TMEM so that it overlaps the next item's
//              main loop), gate_up: SwiGLU and the activation split of h for the down
//              GEMM; down: the routing weight, into the pair's row of ys (a build with
//              MOE_GEMV_FUSE_COMBINE=1 also combines y = x + sum_j w_j o_j there for
//              small batches; by default the combine is its own pass).
// Gate_up weights are stored in 128-row tiles of 64 gate rows (TMEM lanes 0..63) and the
// 64 matching up rows (lanes 64..127), so g and u of one feature meet in the epilogue.
//
// Every wait is bounded (kWaitLimitNs).  When one gives up, the CTA raises its abort
// flag, every role leaves its loop, in-flight copies and MMAs are drained (bounded),
// TMEM is freed and MOE_ERR_TIMEOUT is recorded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;                          // weight rows per tile (TMEM lanes)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: a stuck pipeline, not a slow one

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct MxParams {
  const Tile* tiles;
  const int32_t* ntiles;
  const uint8_t* w_sf;     // weight scale-factor groups [E][NT][KC][512]
  const uint8_t* bp_in;    // packed activation blocks of this GEMM [tiles][KC][block]
  int32_t NT;              // 128-row tiles per expert
  int32_t K;               // reduction length (d for gate_up, I for down)
  int32_t KC;              // 128-chunks of the reduction axis (K rounded up)
  int32_t n_rt;            // row tiles per token tile: I/64 (gate_up) or ceil(d/128) (down)
  int32_t n_ru;            // row units per token tile: n_rt, or ceil(n_rt / 2) for CTA pairs
  int32_t ksplit_max;      // reduction-axis splits per (token tile, row tile) allowed (down only)
  int32_t* ksplit_out;     // down: the number of splits used (the planes of ys the combine adds)
  int32_t P;               // pairs (rows of ys per split)
  int32_t* status;
  float limit;
  int32_t inject_timeout;  // test hook: CTA 0 withholds its first stage
  // gate_up output: h as packed activation blocks of the down GEMM [tiles][KCo][block]
  uint8_t* bp_out;
  int32_t KCo;             // 128-chunks of I
  // down output: ys [ksplit][P][d] fp32 = w * (partial) o, row t * k + slot; optionally
  // y = bf16(x + sum_j sum_s ys[s][t*k + j]) by the last writer of each (token,
  // 128-column) block
  float* ys;
  int32_t d;
  const float* w_sorted;
  int32_t fuse_combine;
  int32_t k;
  const int32_t* perm;
  const int32_t* inv;
  const uint16_t* x;
  uint16_t* y;
  float* y_partial;        // instead of y: the fp32 sum without the residual (a slice of I)
  int32_t* arrivals;
  // buffer ends for the stores at computed offsets (bounds-checking builds)
  const uint8_t* bp_out_end;
  const float* ys_end;
  const uint16_t* y_end;
  const float* y_partial_end;
};

#ifndef MOE_SF_SLOTS
#define MOE_SF_SLOTS 2
#endif
constexpr int kSfSlots = MOE_SF_SLOTS;  // scale-factor TMEM slots, used stage after stage in turn

template <int BN, int NP, int S, int CPS, int EG, int NPW, int TERMS, bool FP4, int CG>
struct MxCfg {
  static constexpr int N2 = TERMS * BN;                 // MMA N: hi (and lo) column per token
  static constexpr int G = (N2 + 127) / 128;            // scale-factor groups of the B operand
  // Bytes of one operand row of a 128-chunk: E2M1 unpacked to a byte per code (A) or E4M3
  // (B), 128; with MXFP4 activations both operands are packed E2M1, 64.
  static constexpr int RB = FP4 ? kKChunk / 2 : kKChunk;
  static constexpr int A_PANEL = kBM * RB;              // 128 weight rows
  static constexpr int B_BLOCK = packed_block_bytes(N2, RB);  // B panel + its scale factors, padded
  // A CTA pair (CG = 2) shares one MMA of M = 256: each CTA holds its 128 weight rows, half
  // of the B rows and all of B's scale factors; one chunk per stage.
  static constexpr int B_ROWS = N2 / CG;                // B rows in this CTA's shared memory
  static constexpr int B_SF_OFF = B_ROWS * RB;          // B's scale factors within a chunk's B region
  static constexpr int B_SMEM = CG == 1 ? B_BLOCK : ((B_SF_OFF + G * kSfGroupBytes + 1023) / 1024) * 1024;
  static constexpr int B_OFF = NP * A_PANEL;
  static constexpr int SFA_OFF = B_OFF + NP * B_SMEM;
  static constexpr int STAGE_BYTES = ((SFA_OFF + NP * kSfGroupBytes + 1023) / 1024) * 1024;
  static constexpr int A_TX = NP * kBM * kKChunk / 2;   // the weight box counts packed bytes
  static constexpr int PAIR_TX = A_TX + B_SF_OFF + G * kSfGroupBytes + kSfGroupBytes;  // one CTA's stage (pairs)
  static constexpr int CW = N2 < 32 ? N2 : 32;          // accumulator columns per epilogue read
  static constexpr int TC = CW / TERMS;                 // tokens per epilogue read
  static constexpr int SB = 8;                          // tokens per g / u exchange round (gate_up)
  static constexpr int ACC_COLS = N2 < 32 ? 32 : N2;    // one accumulator buffer
  static constexpr int SF_SLOT_COLS = 4 * NP * (1 + G);         // A then B scale factors of a stage
  static constexpr int SFA_COL = 2 * ACC_COLS;                   // + slot * SF_SLOT_COLS
  static constexpr int SFB_COL = SFA_COL + 4 * NP;
  static constexpr int COLS_NEEDED = 2 * ACC_COLS + kSfSlots * SF_SLOT_COLS;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 32 ? 32 : COLS_NEEDED <= 64 ? 64 : COLS_NEEDED <= 128 ? 128
                                   : COLS_NEEDED <= 256 ? 256 : 512;
  // two buffers of g and u of SB tokens (gate_up), then the token list (down)
  static constexpr int EPI_GROUP_BYTES = 4 * SB * 64 * 4 + TC * 4;
  static constexpr int EPI_BYTES = EG * EPI_GROUP_BYTES;
  // barriers per stage: one per copy issuer (pairs: one, the leader's, for all copies)
  static constexpr int NISS = CG == 2 ? 1 : NPW;
  static constexpr int BAR_BYTES = 8 * ((NISS + 1) * S + 5) + 16;
  static constexpr int SMEM_BYTES = S * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024 /*align slack*/;
  static constexpr int EPI_THREADS = 128 * EG;
  static constexpr int MMA_WARP = NPW;                // warps 0..NPW-1 produce
  static constexpr int EPI_WARP0 = NPW + 1;
  static constexpr int THREADS = 32 * EPI_WARP0 + EPI_THREADS;
  static_assert(N2 == 16 || (N2 % 32 == 0 && N2 <= 256), "MMA N: 16 or a multiple of 32 up to 256");
  static_assert(COLS_NEEDED <= 512 && TMEM_COLS * CPS <= 512, "TMEM budget of CPS co-resident CTAs");
  static_assert(SMEM_BYTES * CPS <= 227 * 1024, "shared memory budget of CPS co-resident CTAs");
  static_assert(kBM * NP <= 256, "TMA box height");
  static_assert(EG >= 1 && EG <= 3, "one to three epilogue warpgroups");
  static_assert(CG == 1 || (CG == 2 && NP == 1 && CPS == 1 && B_ROWS % 8 == 0),
                "CTA pairs: one chunk per stage, one CTA per SM");
  static_assert(TC % SB == 0, "an epilogue read holds whole exchange rounds");
  static_assert(NPW >= 1 && NPW <= (CG == 2 ? 4 : 3), "producer warps: one per kind of copy at most");
};

// Work item i: token tile tt, row tile rt, and the chunk range [kc0, kc1) of split ks.
struct Item {
  int tt, rt, ks, kc0, kc1;
};

__device__ __forceinline__ Item item_of(const MxParams& p, int i, int ksplit, int cg, int rank) {
  Item it;
  const int r = i / ksplit;
  it.ks = i - r * ksplit;
  it.tt = r / p.n_ru;
  it.rt = cg * (r - it.tt * p.n_ru) + rank;   // a pair's CTAs take consecutive row tiles
  it.kc0 = it.ks * p.KC / ksplit;
  it.kc1 = (it.ks + 1) * p.KC / ksplit;
  return it;
}

// Accumulator of token j in a 32-column epilogue read: the sum of its hi and lo columns
// (bf16 activations carried as two E4M3 terms) or its one column (MXFP8 activations).
template <int TERMS>
__device__ __forceinline__ float token_acc(const uint32_t (&v)[32], int j) {
  if (TERMS == 2) return __uint_as_float(v[2 * j]) + __uint_as_float(v[2 * j + 1]);
  return __uint_as_float(v[j]);
}

// Splits of the reduction axis for n0 (token tile, row tile) units over `grid` CTAs: the
// count (at most smax) that minimises the busiest CTA's work, ceil(n0 ks / grid) items of
// 1 / ks of a unit each plus a fixed cost per item (its epilogue and pipeline turn-around,
// taken as 1/16 of a whole unit); a CTA with a single item has no next item's loads to
// hide that item's epilogue under (the accumulator is double-buffered), which counts as
// one more unit.  Ties go to fewer splits.
__device__ __forceinline__ int choose_ksplit(int n0, int grid, int smax) {
  if (n0 <= 0 || smax <= 1) return 1;
  int best = 1;
  float best_t = 3.4e38f;
  for (int ks = 1; ks <= smax; ++ks) {
    const int per_cta = (n0 * ks + grid - 1) / grid;
    const float t = (float)per_cta * (1.0f / (float)ks + 0.0625f) + (per_cta < 2 ? 1.0f : 0.f);
    if (t < best_t - 1e-6f) {
      best_t = t;
      best = ks;
    }
  }
  return best;
}

// The tcgen05 operations of one CTA (CG = 1) or of a CTA pair issued by its leader (CG = 2).
template <int CG>
__device__ __forceinline__ void cp_sf(uint32_t taddr, uint64_t desc) {
  if (CG == 2) ptx::tc_cp_32x128b_x4_pair(taddr, desc);
  else ptx::tc_cp_32x128b_x4(taddr, desc);
}
template <int CG>
__device__ __forceinline__ void mma_f8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t acc) {
  if (CG == 2) ptx::mma_mx_ss_pair(d, a, b, idesc, sfa, sfb, acc);
  else ptx::mma_mx_ss(d, a, b, idesc, sfa, sfb, acc);
}
template <int CG>
__device__ __forceinline__ void mma_f4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t acc) {
  if (CG == 2) ptx::mma_mxf4_ss_pair(d, a, b, idesc, sfa, sfb, acc);
  else ptx::mma_mxf4_ss(d, a, b, idesc, sfa, sfb, acc);
}
// Arrive on `bar` (in both CTAs of a pair) when the issued tcgen05 operations are done.
template <int CG>
__device__ __forceinline__ void commit_to(uint64_t* bar) {
  if (CG == 2) ptx::tc_commit_pair(bar, (uint16_t)0x3);
  else ptx::tc_commit(bar);
}

template <int BN, int NP, int S, int CPS, int EG, int NPW, int TERMS, bool FP4, int CG, int MODE>
__global__ void __launch_bounds__(MxCfg<BN, NP, S, CPS, EG, NPW, TERMS, FP4, CG>::THREADS, CPS)
    mx_expert_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_bsf, const __grid_constant__ CUtensorMap tm_sfa,
                     const MxParams p) {
  using C = MxCfg<BN, NP, S, CPS, EG, NPW, TERMS, FP4, CG>;
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + S * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + C::EPI_BYTES);   // [S][NISS] copies landed
  uint64_t* sfree = full + S * C::NISS;   // stage consumed (its MMAs done)
  uint64_t* accf = sfree + S;       // [2] accumulator ready
  uint64_t* acce = accf + 2;        // [2] accumulator drained by the epilogue
  uint64_t* drain = acce + 2;       // final MMA drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = p.K / 32;
  // CTA pairs: rank 0 (the leader) issues the MMAs; both CTAs walk the same items
  const int rank = CG == 2 ? (int)ptx::cluster_ctarank() : 0;
  const int unit0 = CG == 2 ? (int)blockIdx.x / 2 : (int)blockIdx.x;
  const int unit_stride = CG == 2 ? (int)gridDim.x / 2 : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      for (int w = 0; w < C::NISS; ++w) ptx::mbar_init(&full[s * C::NISS + w], 1);
      ptx::mbar_init(&sfree[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&accf[b], 1);
      // drained by every epilogue thread; with pairs, by one lane per epilogue warp of each CTA
      ptx::mbar_init(&acce[b], CG == 2 ? CG * (C::EPI_THREADS / 32) : C::EPI_THREADS);
    }
    ptx::mbar_init(drain, 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tm_w);
    if (CG == 2) {
      ptx::prefetch_tensormap(&tm_b);
      ptx::prefetch_tensormap(&tm_bsf);
      ptx::prefetch_tensormap(&tm_sfa);
    }
  }
  if (warp == C::MMA_WARP) {
    if (CG == 2) {
      ptx::tmem_alloc_pair(s_tmem, C::TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(s_tmem, C::TMEM_COLS);
      ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
  }
  // (pairs: the peer's copies, commits and arrivals find initialized barriers)
  if (CG == 2) ptx::cluster_sync();
  else __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // Everything above overlaps the previous kernel; the work list is its output.
  pdl_wait();
  const int n_units = *p.ntiles * p.n_ru;
  const int ksplit = choose_ksplit(n_units, unit_stride, p.ksplit_max);   // same in every CTA
  const int n_items = n_units * ksplit;
  if (MODE == MODE_DOWN && blockIdx.x == 0 && threadIdx.x == 0) *p.ksplit_out = ksplit;

  auto a_s = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto b_s = [&](int s) { return smem + s * C::STAGE_BYTES + C::B_OFF; };
  auto sfa_s = [&](int s) { return smem + s * C::STAGE_BYTES + C::SFA_OFF; };

  if (warp < NPW) {
    // ------------------------------------------------------------------ producers
    // Every stage takes three copies: the weight box (TMA), the activation block and the
    // weight scale factors (bulk).  Producer warp w issues the kinds k with k % NPW == w on
    // its own barrier full[s][w], so that one warp's copies do not queue behind another's;
    // the warp waits converged and lane 0 issues.
    int64_t g = 0;  // global stage counter of this CTA
    bool stop = false, withheld = false;
    for (int i = unit0; i < n_items && !stop; i += unit_stride) {
      const Item it = item_of(p, i, ksplit, CG, rank);
      const int tt = it.tt, rt = it.rt;
      const int nst = (it.kc1 - it.kc0 + NP - 1) / NP;   // stages of this item
      const Tile tl = p.tiles[tt];
      for (int st = 0; st < nst; ++st, ++g) {
        const int s = (int)(g % S);
        bool ok = true;
        if (g >= S) ok = ptx::mbar_wait_bounded(&sfree[s], (uint32_t)((g / S) - 1) & 1, s_abort, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
          stop = true;
          break;
        }
        if (p.inject_timeout && blockIdx.x == 0 && g == 0) {
          withheld = true;  // this stage never fills: the MMA issuer's wait gives up
          continue;
        }
        const int c0 = it.kc0 + st * NP, nck = min(NP, it.kc1 - c0);
        if (CG == 2) {
          // Pairs: this CTA's weight rows (row tile rt; a pair's tile past the last re-reads
          // the last, its results are not stored), its half of the token tile's B rows, all
          // of B's scale factors and its weight scale factors, completing on the leader's
          // barrier, which expects both CTAs' bytes.
          // (several producer warps: warp w issues the copies k with k % NPW == w; the
          // leader's warp 0 posts the byte count of all of them)
          if (ptx::elect_one()) {
            const uint32_t bar = ptx::mapa_shared(&full[s], 0);
            if (rank == 0 && warp == 0) ptx::mbar_arrive_expect_tx(&full[s], CG * C::PAIR_TX);
            const int rt_ld = min(rt, p.NT - 1);
            const int64_t wrow = (((int64_t)tl.e * p.NT + rt_ld) * p.KC + c0);
            const int64_t brow = ((int64_t)tt * p.KC + c0) * (C::B_BLOCK / C::RB);   // rows of RB bytes
            if (0 % NPW == warp) ptx::tma_load_2d_pair(a_s(s), &tm_w, 0, (int)(wrow * kBM), bar);
            if (1 % NPW == warp) ptx::tma_load_2d_pair(b_s(s), &tm_b, 0, (int)(brow + rank * C::B_ROWS), bar);
            if (2 % NPW == warp) ptx::tma_load_2d_pair(b_s(s) + C::B_SF_OFF, &tm_bsf, 0, (int)(brow + C::N2), bar);
            if (3 % NPW == warp)
              ptx::tma_load_2d_pair(sfa_s(s), &tm_sfa, 0, (int)(wrow * (kSfGroupBytes / 128)), bar);
          }
          __syncwarp();
          continue;
        }
        if (ptx::elect_one()) {
          uint64_t* bar = &full[s * C::NISS + warp];
          const bool do_w = (0 % NPW) == warp, do_b = (1 % NPW) == warp, do_f = (2 % NPW) == warp;
          ptx::mbar_arrive_expect_tx(bar, (do_w ? C::A_TX : 0) + (do_b ? nck * C::B_BLOCK : 0) +
                                              (do_f ? nck * kSfGroupBytes : 0));
          if (do_w)
            ptx::tma_load_2d(a_s(s), &tm_w, 0, (int)(((int64_t)tl.e * p.NT + rt) * p.KC + c0) * kBM, bar);
          if (do_b) ptx::bulk_load(b_s(s), p.bp_in + ((int64_t)tt * p.KC + c0) * C::B_BLOCK, nck * C::B_BLOCK, bar);
          if (do_f)
            ptx::bulk_load(sfa_s(s), p.w_sf + ((int64_t)(tl.e * p.NT + rt) * p.KC + c0) * kSfGroupBytes,
                           nck * kSfGroupBytes, bar);
        }
        __syncwarp();
      }
    }
    // Never leave copies in flight when the CTA exits (consumers may have aborted before
    // waiting for them): wait, bounded, for this warp's last fill of every slot.  On the
    // normal path these have all landed already.
    // (pairs: both CTAs' copies complete on the leader's barriers; the leader waits for
    // them here and the cluster barrier at the end holds the peer until it has)
    if (CG == 1 || (rank == 0 && warp == 0)) {
      volatile int local_abort = 0;
      for (int64_t q = (g > S ? g - S : 0); q < g; ++q) {
        if (withheld && q == 0) continue;
        ptx::mbar_wait_bounded(&full[(q % S) * C::NISS + warp], (uint32_t)(q / S) & 1, &local_abort, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    // The warp waits converged; one elected lane issues the copies into TMEM, the MMAs and
    // the commits.  With CTA pairs only the leader's issuer runs the loop; the commits reach
    // the barriers of both CTAs.
    if (CG == 1 || rank == 0) {
      int64_t g = 0;
      int li = 0;
      bool stop = false;
      for (int i = unit0; i < n_items && !stop; i += unit_stride, ++li) {
        const int b = li & 1;
        // (pairs: the drain arrivals come from the epilogues of both CTAs)
        if (li >= 2 &&
            !__all_sync(0xffffffffu,
                        CG == 2 ? ptx::mbar_wait_cluster_bounded(&acce[b], (uint32_t)((li >> 1) - 1) & 1, s_abort,
                                                                 kWaitLimitNs)
                                : ptx::mbar_wait_bounded(&acce[b], (uint32_t)((li >> 1) - 1) & 1, s_abort,
                                                         kWaitLimitNs)))
          break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + b * C::ACC_COLS;
        const Item it = item_of(p, i, ksplit, CG, rank);
        const int nst = (it.kc1 - it.kc0 + NP - 1) / NP;
        for (int st = 0; st < nst; ++st, ++g) {
          const int s = (int)(g % S);
          bool landed = true;
          for (int w = 0; w < C::NISS && landed; ++w)
            landed = ptx::mbar_wait_bounded(&full[s * C::NISS + w], (uint32_t)(g / S) & 1, s_abort, kWaitLimitNs);
          if (!__all_sync(0xffffffffu, landed)) {
            stop = true;
            break;
          }
          ptx::tc_fence_after();
          const int c0 = it.kc0 + st * NP, nck = min(NP, it.kc1 - c0);
          if (ptx::elect_one()) {
            // scale factors of this stage into their TMEM slot (the tensor pipe runs one
            // thread's copies and MMAs in issue order; with two slots a copy does not
            // overwrite columns the previous stage's MMAs still read)
            const uint32_t sf_slot = tmem + (uint32_t)((g % kSfSlots) * C::SF_SLOT_COLS);
            const uint64_t a0 = FP4 ? ptx::smem_desc_k_sw64(a_s(s)) : ptx::smem_desc_k_sw128(a_s(s));
            const uint64_t b0 = FP4 ? ptx::smem_desc_k_sw64(b_s(s)) : ptx::smem_desc_k_sw128(b_s(s));
            const uint64_t f0 = ptx::smem_desc_k_rows16(sfa_s(s)), fb0 = ptx::smem_desc_k_rows16(b_s(s) + C::B_SF_OFF);
            // (descriptor start addresses count 16-byte units: offsets within shared memory add)
            constexpr uint64_t kA = C::A_PANEL >> 4, kB = C::B_SMEM >> 4, kF = kSfGroupBytes >> 4;
            if (nck == NP && 4 * (c0 + NP) <= kblocks) {
              // a full stage: NP chunks of 4 blocks of 32, every index a compile-time constant
#pragma unroll
              for (int c = 0; c < NP; ++c) {
                cp_sf<CG>(sf_slot + C::SFA_COL + 4 * c, f0 + c * kF);
#pragma unroll
                for (int gg = 0; gg < C::G; ++gg)
                  cp_sf<CG>(sf_slot + C::SFB_COL + 4 * (c * C::G + gg), fb0 + c * kB + gg * kF);
              }
#pragma unroll
              for (int c = 0; c < NP; ++c) {
                const uint32_t sfa = sf_slot + C::SFA_COL + 4 * c, sfb = sf_slot + C::SFB_COL + 4 * c * C::G;
                if (FP4) {
#pragma unroll
                  for (int kk = 0; kk < 2; ++kk)
                    mma_f4<CG>(d_tmem, a0 + c * kA + 2 * kk, b0 + c * kB + 2 * kk,
                                     ptx::idesc_mxf4(kBM * CG, C::N2, (uint32_t)(2 * kk), (uint32_t)(2 * kk)), sfa, sfb,
                                     (st | c | kk) != 0);
                } else {
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk)
                    mma_f8<CG>(d_tmem, a0 + c * kA + 2 * kk, b0 + c * kB + 2 * kk,
                                   ptx::idesc_mx_e2m1_e4m3(kBM * CG, C::N2, (uint32_t)kk, (uint32_t)kk), sfa, sfb,
                                   (st | c | kk) != 0);
                }
              }
            } else {
              for (int c = 0; c < nck; ++c) {
                cp_sf<CG>(sf_slot + C::SFA_COL + 4 * c, f0 + c * kF);
#pragma unroll
                for (int gg = 0; gg < C::G; ++gg)
                  cp_sf<CG>(sf_slot + C::SFB_COL + 4 * (c * C::G + gg), fb0 + c * kB + gg * kF);
              }
              for (int c = 0; c < nck; ++c) {
                const int nkb = min(4, kblocks - 4 * (c0 + c));   // 32-blocks of this chunk (K % 64 == 0: even)
                const uint32_t sfa = sf_slot + C::SFA_COL + 4 * c, sfb = sf_slot + C::SFB_COL + 4 * c * C::G;
                if (FP4) {
                  // FP4 x FP4: one MMA per 64 k (32 bytes of each packed row); it takes the scale
                  // bytes 2kk and 2kk + 1 of each row's scale-factor word
                  for (int kk = 0; kk < nkb / 2; ++kk)
                    mma_f4<CG>(d_tmem, a0 + c * kA + 2 * kk, b0 + c * kB + 2 * kk,
                                     ptx::idesc_mxf4(kBM * CG, C::N2, (uint32_t)(2 * kk), (uint32_t)(2 * kk)), sfa, sfb,
                                     (st | c | kk) != 0);
                } else {
                  // E2M1 x E4M3: one MMA per 32 k (32 bytes of each row), scale byte kk
                  for (int kk = 0; kk < nkb; ++kk)
                    mma_f8<CG>(d_tmem, a0 + c * kA + 2 * kk, b0 + c * kB + 2 * kk,
                                   ptx::idesc_mx_e2m1_e4m3(kBM * CG, C::N2, (uint32_t)kk, (uint32_t)kk), sfa, sfb,
                                   (st | c | kk) != 0);
                }
              }
            }
            commit_to<CG>(&sfree[s]);
          }
          __syncwarp();
        }
        if (!stop && ptx::elect_one()) commit_to<CG>(&accf[b]);
        __syncwarp();
      }
      // Every MMA issued above completes before the drain barrier fires (in both CTAs).
      if (ptx::elect_one()) commit_to<CG>(drain);
      __syncwarp();
    }
    {
      volatile int local_abort = 0;
      ptx::mbar_wait_bounded(drain, 0, &local_abort, kWaitLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;       // weight row of the tile == TMEM lane
    const int eg = (warp - C::EPI_WARP0) >> 2;   // epilogue warpgroup: reads c0 = (eg + EG*m) * CW
    const int et = threadIdx.x - 32 * C::EPI_WARP0 - 128 * eg;  // 0..127 within the group
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    uint8_t* gepi = epi + eg * C::EPI_GROUP_BYTES;
    // The accumulator buffer goes back to the MMA issuer (pairs: one arrival per warp on the
    // leader's barrier, after every lane's TMEM reads)
    auto release_acc = [&](int b) {
      ptx::tc_fence_before();
      if (CG == 2) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(&acce[b], 0));
      } else {
        ptx::mbar_arrive(&acce[b]);
      }
    };
    auto group_sync = [&]() {            // the group's named barrier (128 threads; 3 is the epilogue-wide vote)
      if (eg == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
      else if (eg == 1) asm volatile("bar.sync 2, 128;" ::: "memory");
      else asm volatile("bar.sync 4, 128;" ::: "memory");
    };
    int li = 0;
    int rnd = 0;   // g / u exchange rounds so far (gate_up)
    for (int i = unit0; i < n_items; i += unit_stride, ++li) {
      const int b = li & 1;
      const bool ready = !*s_abort && ptx::mbar_wait_bounded(&accf[b], (uint32_t)(li >> 1) & 1, s_abort,
                                                             kWaitLimitNs);
      // All epilogue warps take the same branch (the abort flag may be raised by another
      // role at any time; the barrier reduction freezes one answer for all).
      if (ptx::bar_or<3, C::EPI_THREADS>(!ready)) break;
      ptx::tc_fence_after();
      const Item it = item_of(p, i, ksplit, CG, rank);
      const int tt = it.tt, rt = it.rt;
      const Tile tl = p.tiles[tt];
      const uint32_t acc = tmem + lane_addr + b * C::ACC_COLS;
      if (MODE == MODE_GATE_UP) {
        // Per read of TC tokens, in rounds of SB tokens: the gate threads (lane rows 0..63)
        // put g, the up threads (rows 64..127) put u into shared memory; then each thread
        // finishes 4 consecutive features of one token: h = bf16(silu(g) * u) and its share
        // of the down GEMM's activation block (8 threads per 32-feature block: E4M3 hi / lo
        // terms and their scales, the hi term alone with MXFP8 activations, or E2M1 codes).
        // (two exchange buffers used round after round: a round's writes go to the buffer
        // last read two rounds before, which the previous round's barrier has released)
        float* const s_gu = reinterpret_cast<float*>(gepi);  // [2][g, u][SB tokens][64 features]
        const float L = p.limit;
        const int f = 32 * (q & 1) + lane;           // feature within the item's 64
        const int jj = et >> 4;                      // token of the round this thread finishes
        const int bq = (et >> 3) & 1;                // its 32-feature block (of the item's two)
        const int u = et & 7;                        // features 32 bq + 4 u .. + 3
        const int kb = 2 * rt + bq;                  // the block along the down GEMM's K
        if (eg * C::CW >= C::N2) {  // nothing for this group to read
          release_acc(b);
        }
        for (int c0 = eg * C::CW; c0 < C::N2; c0 += EG * C::CW) {
          uint32_t v[32];
          ptx::tmem_ld32(acc + c0, v);
          ptx::tmem_wait_ld();
          if (c0 + EG * C::CW >= C::N2) {  // last read: the accumulator goes back to the MMA issuer
            release_acc(b);
          }
#pragma unroll
          for (int sb = 0; sb < C::TC; sb += C::SB) {
            // (register indices stay compile-time constants)
            float* s_g = s_gu + (rnd & 1) * 2 * C::SB * 64;
            float* s_u = s_g + C::SB * 64;
            float* s_mine = (q < 2) ? s_g : s_u;
            ++rnd;
#pragma unroll
            for (int c = 0; c < C::SB; ++c) s_mine[c * 64 + f] = token_acc<TERMS>(v, sb + c);
            group_sync();
            const float4 g4 = *reinterpret_cast<const float4*>(s_g + jj * 64 + 32 * bq + 4 * u);
            const float4 u4 = *reinterpret_cast<const float4*>(s_u + jj * 64 + 32 * bq + 4 * u);
            const float gs[4] = {g4.x, g4.y, g4.z, g4.w}, us[4] = {u4.x, u4.y, u4.z, u4.w};
            float hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float gv = fminf(gs[i], L);
              const float uv = fminf(fmaxf(us[i], -L), L);
              const float h = __fdividef(gv, 1.0f + __expf(-gv)) * uv;   // silu(g) * u
              hv[i] = __bfloat162float(__float2bfloat16_rn(h));   // h is stored as bf16 (round to nearest even)
            }
            const int j = c0 / TERMS + sb + jj;   // token within the tile
            uint8_t* blk = p.bp_out + ((int64_t)tt * p.KCo + kb / 4) * C::B_BLOCK;
            if (FP4) {
              // MXFP4 activations: 4 E2M1 codes (2 bytes) of row j's 64-byte row, unit kb % 4
              uint32_t codes, sf4;
              e2m1_quant<4>(hv, codes, sf4);
              if (j < tl.rows && rt < p.n_rt) {
                uint16_t* q2 = reinterpret_cast<uint16_t*>(blk + packed_unit_offset64(j, kb & 3) + 2 * u);
                if (in_bounds(q2, p.bp_out, p.bp_out_end, p.status)) *q2 = (uint16_t)codes;
                uint8_t* qs = blk + packed_sf_offset(C::N2, j, kb, C::RB);
                if (u == 0 && in_bounds(qs, p.bp_out, p.bp_out_end, p.status)) *qs = (uint8_t)sf4;
              }
            } else {
              uint32_t hi, lo, s1, s2;
              e4m3_split<4>(hv, hi, lo, s1, s2);
              if (j < tl.rows && rt < p.n_rt) {
                // the down GEMM's packed block: chunk kb / 4, rows TERMS j (hi) and 2 j + 1 (lo),
                // bytes 32 (kb % 4) + 4 u .. + 3 of the 128-byte row
                const int unit = 2 * (kb & 3) + (u >> 2);
                uint32_t* qh = reinterpret_cast<uint32_t*>(blk + packed_unit_offset(TERMS * j, unit) + 4 * (u & 3));
                if (in_bounds(qh, p.bp_out, p.bp_out_end, p.status)) *qh = hi;
                uint32_t* ql = reinterpret_cast<uint32_t*>(blk + packed_unit_offset(2 * j + 1, unit) + 4 * (u & 3));
                if (TERMS == 2 && in_bounds(ql, p.bp_out, p.bp_out_end, p.status)) *ql = lo;
                if (u == 0) {
                  uint8_t* qs = blk + packed_sf_offset(C::N2, TERMS * j, kb);
                  if (in_bounds(qs, p.bp_out, p.bp_out_end, p.status)) *qs = (uint8_t)s1;
                  qs = blk + packed_sf_offset(C::N2, 2 * j + 1, kb);
                  if (TERMS == 2 && in_bounds(qs, p.bp_out, p.bp_out_end, p.status)) *qs = (uint8_t)s2;
                }
              }
            }
          }
        }
      } else {
        int* s_tok = reinterpret_cast<int*>(gepi + 4 * C::SB * 64 * 4);  // [TC]
        float* ys = p.ys + (int64_t)it.ks * p.P * p.d;               // this split's partial sums
        const int m = kBM * rt + row;                                // output feature
        const int ncol = min(kBM, p.d - kBM * rt);
        if (eg * C::CW >= C::N2) {
          release_acc(b);
        }
        for (int c0 = eg * C::CW; c0 < C::N2; c0 += EG * C::CW) {
          uint32_t v[32];
          ptx::tmem_ld32(acc + c0, v);
          ptx::tmem_wait_ld();
          if (c0 + EG * C::CW >= C::N2) {
            release_acc(b);
          }
          const int jbase = c0 / TERMS;
          const int nt = min(C::TC, tl.rows - jbase);   // tokens of this read (may be <= 0)
#pragma unroll
          for (int c = 0; c < C::TC; ++c) {
            if (c < nt && m < p.d) {
              const int64_t prow = tl.row0 + jbase + c;
              const float o = token_acc<TERMS>(v, c);
              // the row of pair t * k + slot: each token's k outputs are consecutive rows
              float* q = ys + (int64_t)__ldg(p.perm + prow) * p.d + m;
              if (in_bounds(q, p.ys, p.ys_end, p.status)) *q = o * p.w_sorted[prow];
            }
          }
          if (CG == 1 && p.fuse_combine) {
            // Publish this read's outputs, count them per (token, column block); the writer of
            // a token's k-th contribution adds the k outputs in slot order plus the residual.
            __threadfence();
            group_sync();
            if (et < nt) {
              const int tok = p.perm[tl.row0 + jbase + et] / p.k;
              const int prev = atomicAdd(p.arrivals + (int64_t)tok * p.n_rt + rt, 1);
              s_tok[et] = (prev == p.k * ksplit - 1) ? tok : -1;
            }
            group_sync();
            __threadfence();
            for (int t = 0; t < nt; ++t) {
              const int tok = s_tok[t];
              if (tok < 0) continue;
              for (int col = et; col < ncol; col += 128) {
                const int64_t gc = kBM * rt + col;
                float accv = p.y_partial ? 0.f : __uint_as_float((uint32_t)p.x[(int64_t)tok * p.d + gc] << 16);
                constexpr int kMaxParts = 24;   // k x splits loaded together (else one after another)
                if (p.k * ksplit <= kMaxParts) {
                  // every partial row's position first, then all their loads in flight at once;
                  // the sum keeps the order slot, then split
                  int srow[kMaxParts];
                  float part[kMaxParts];
#pragma unroll
                  for (int q = 0; q < kMaxParts; ++q)   // part q: slot q / ksplit, split q % ksplit
                    if (q < p.k * ksplit) srow[q] = tok * p.k + q / ksplit;
#pragma unroll
                  for (int q = 0; q < kMaxParts; ++q)
                    if (q < p.k * ksplit)
                      part[q] = __ldcg(p.ys + ((int64_t)(q % ksplit) * p.P + srow[q]) * p.d + gc);
#pragma unroll
                  for (int q = 0; q < kMaxParts; ++q)
                    if (q < p.k * ksplit) accv += part[q];
                } else {
                  for (int j = 0; j < p.k; ++j) {
                    const int srow1 = tok * p.k + j;
                    for (int sp = 0; sp < ksplit; ++sp)
                      accv += __ldcg(p.ys + ((int64_t)sp * p.P + srow1) * p.d + gc);
                  }
                }
                if (p.y_partial) {
                  float* q = p.y_partial + (int64_t)tok * p.d + gc;
                  if (in_bounds(q, p.y_partial, p.y_partial_end, p.status)) *q = accv;
                } else {
                  uint16_t* q = p.y + (int64_t)tok * p.d + gc;
                  if (in_bounds(q, p.y, p.y_end, p.status)) *q = bf16_bits_rne(accv);
                }
              }
            }
            group_sync();
          }
        }
      }
    }
  }

  __syncthreads();
  if (*s_abort && threadIdx.x == 0) set_status(p.status, MOE_ERR_TIMEOUT);
  // (pairs: the leader has seen every copy of both CTAs land and the MMAs into both TMEMs
  // complete before either CTA frees its TMEM and exits)
  if (CG == 2) ptx::cluster_sync();
  if (warp == C::MMA_WARP) {
    ptx::tc_fence_after();
    if (CG == 2) ptx::tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else ptx::tmem_dealloc(tmem, C::TMEM_COLS);
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
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[4], gs[3];
  cuuint32_t bx[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  return fn(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Clusters of two CTAs of `kern` that fit on the device at once (0 if none or on error).
template <class K>
int max_pair_clusters(K kern, int threads, int smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * sm_count());
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

template <int MODE, int BN, int NP, int S, int CPS, int EG, int NPW, int TERMS, bool FP4, int KSPLIT, int CG = 1>
int launch_one(const FwdArgs& a) {
  using C = MxCfg<BN, NP, S, CPS, EG, NPW, TERMS, FP4, CG>;
  const int P = a.T * a.k;
  const int K = (MODE == MODE_GATE_UP) ? a.d : a.I;
  const int N = (MODE == MODE_GATE_UP) ? 2 * a.I : a.d;  // weight rows per expert
  const int64_t Kp = kpad128(K);
  const int KC = (int)(Kp / kKChunk);
  const uint8_t* codes = (MODE == MODE_GATE_UP) ? a.w1c : a.w2c;
  const uint8_t* scales = (MODE == MODE_GATE_UP) ? a.w1s : a.w2s;

  // Weight codes [E][NT][KC][128][64] viewed as rows of 64 bytes: one box brings NP
  // consecutive tile blocks (NP x 128 rows).  E2M1 x E4M3: the rows are 128 codes, unpacked
  // by the copy to a byte each, 128B-swizzled [128][128] panels in shared memory; FP4 x FP4:
  // the packed bytes as stored, 64B-swizzled [128][64] panels.
  CUtensorMap m_w;
  {
    const int NT = (N + kBM - 1) / kBM;
    const uint64_t rows = (uint64_t)a.E * NT * KC * kBM;
    const uint64_t str[1] = {(uint64_t)kKChunk / 2};
    if (FP4) {
      const uint64_t dims[2] = {(uint64_t)kKChunk / 2, rows};
      const uint32_t box[2] = {kKChunk / 2, (uint32_t)(kBM * NP)};
      if (!make_map(&m_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
        return -1;
    } else {
      const uint64_t dims[2] = {(uint64_t)kKChunk, rows};
      const uint32_t box[2] = {kKChunk, (uint32_t)(kBM * NP)};
      if (!make_map(&m_w, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, codes, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    }
  }
  // CTA pairs load everything by tile copies that complete on the leader's barrier: the
  // token tile's packed activation blocks viewed as rows of RB bytes (a CTA's half of the B
  // rows; the scale-factor rows after them), and the weight scale factors as 128-byte rows
  // (one 512-byte group per chunk).  The blocks are already in the order the MMA reads.
  CUtensorMap m_b = m_w, m_bsf = m_w, m_sfa = m_w;
  if (CG == 2) {
    const int NT = (N + kBM - 1) / kBM;
    const uint8_t* bp = (MODE == MODE_GATE_UP) ? a.ws.bpx : a.ws.bph;
    const uint64_t brows = (uint64_t)a.ws.max_tiles * KC * (C::B_BLOCK / C::RB);
    const uint64_t bdims[2] = {(uint64_t)C::RB, brows}, bstr[1] = {(uint64_t)C::RB};
    const uint32_t bbox[2] = {(uint32_t)C::RB, (uint32_t)C::B_ROWS};
    const uint32_t sbox[2] = {(uint32_t)C::RB, (uint32_t)(C::G * kSfGroupBytes / C::RB)};
    const uint64_t fdims[2] = {128, (uint64_t)a.E * NT * KC * (kSfGroupBytes / 128)}, fstr[1] = {128};
    const uint32_t fbox[2] = {128, kSfGroupBytes / 128};
    if (!make_map(&m_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, bp, bdims, bstr, bbox, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&m_bsf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, bp, bdims, bstr, sbox, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&m_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, scales, fdims, fstr, fbox, CU_TENSOR_MAP_SWIZZLE_NONE))
      return -1;
  }
  MxParams prm;
  prm.tiles = a.ws.tiles;
  prm.ntiles = a.ws.ntiles;
  prm.w_sf = scales;
  prm.bp_in = (MODE == MODE_GATE_UP) ? a.ws.bpx : a.ws.bph;
  prm.NT = (N + kBM - 1) / kBM;
  prm.K = K;
  prm.KC = KC;
  prm.n_rt = (MODE == MODE_GATE_UP) ? a.I / 64 : (a.d + kBM - 1) / kBM;
  prm.n_ru = (prm.n_rt + CG - 1) / CG;
  prm.ksplit_max = std::max(1, std::min(KSPLIT, KC));   // every split keeps at least one chunk
  prm.ksplit_out = a.ws.ntiles + 1;
  prm.P = P;
  prm.status = a.ws.status;
  prm.limit = a.limit;
  prm.inject_timeout = (MODE == MODE_GATE_UP) ? a.inject_timeout : 0;
  prm.bp_out = a.ws.bph;
  prm.KCo = a.ws.ip / kKChunk;
  prm.ys = a.ws.ys;
  prm.d = a.d;
  prm.w_sorted = a.ws.w_sorted;
  prm.fuse_combine = (MODE == MODE_DOWN) ? a.fuse_combine : 0;
  prm.k = a.k;
  prm.perm = a.ws.perm;
  prm.inv = a.ws.inv;
  prm.x = a.x;
  prm.y = a.y;
  prm.y_partial = a.y_partial;
  prm.bp_out_end = a.ws.bph_end;
  prm.ys_end = a.ws.ys_end;
  prm.y_end = a.y ? a.y + (int64_t)a.T * a.d : nullptr;
  prm.y_partial_end = a.y_partial ? a.y_partial + (int64_t)a.T * a.d : nullptr;
  prm.arrivals = a.ws.arrivals;

  auto kern = mx_expert_kernel<BN, NP, S, CPS, EG, NPW, TERMS, FP4, CG, MODE>;
  static std::atomic<uint64_t> attr_done{0};   // per-device "attribute set" bits
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return -1;
    attr_done.fetch_or(bit, std::memory_order_release);
  }
  const int64_t max_items = (int64_t)((P + BN - 1) / BN + a.E) * prm.n_ru * prm.ksplit_max;
  if (CG == 2) {
    // persistent pairs: as many clusters of two as fit at once
    static std::atomic<int> pair_limit[64];
    int lim = pair_limit[dev & 63].load(std::memory_order_acquire);
    if (lim <= 0) {
      lim = max_pair_clusters(kern, C::THREADS, C::SMEM_BYTES);
      if (lim <= 0) return -1;
      pair_limit[dev & 63].store(lim, std::memory_order_release);
    }
    const int pairs = (int)std::min<int64_t>(max_items, (int64_t)lim);
    ev_before(a);
    if (launch_kernel_cluster(kern, dim3(2 * pairs), dim3(C::THREADS), C::SMEM_BYTES, a.stream, a.pdl != 0, 2u, m_w,
                              m_b, m_bsf, m_sfa, prm) != cudaSuccess)
      return -1;
    ev_after(a);
    return 1;
  }
  const int grid = (int)std::min<int64_t>(max_items, (int64_t)sm_count() * CPS);
  ev_before(a);
  if (launch_kernel(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, a.stream, a.pdl != 0, m_w, m_b, m_bsf, m_sfa,
                    prm) != cudaSuccess)
    return -1;
  ev_after(a);
  return 1;
}

// Pipeline shapes (compile-time; overridable with -D for tuning builds).
// Small batches (few tokens per expert): 8-token tiles (MMA N = 16; 16 tokens with MXFP8
// activations), three independent
// pipelines (CTAs) per SM: each CTA's copies are served in order, so more CTAs keep
// more of HBM's requests in flight.
#ifndef MOE_GEMV_NP
#define MOE_GEMV_NP 1
#endif
#ifndef MOE_GEMV_S
#define MOE_GEMV_S 3
#endif
#ifndef MOE_GEMV_CPS
#define MOE_GEMV_CPS 3
#endif
#ifndef MOE_GEMV_EG
#define MOE_GEMV_EG 1
#endif
#ifndef MOE_GEMV_NPW
#define MOE_GEMV_NPW 1
#endif
#ifndef MOE_GEMV_DOWN_SPLIT
#define MOE_GEMV_DOWN_SPLIT 6
#endif
// Large batches: 96-token tiles (MMA N = 192), one 128-chunk per stage and four stages:
// three stages of copies in flight while one is consumed (16384 tokens x 128 experts:
// gate_up 2.30 ms, down 1.15 ms, against 2.43 / 1.32 ms with two stages of two chunks).
#ifndef MOE_GEMM_NP
#define MOE_GEMM_NP 1
#endif
#ifndef MOE_GEMM_S
#define MOE_GEMM_S 4
#endif
#ifndef MOE_GEMM_CPS
#define MOE_GEMM_CPS 1
#endif
#ifndef MOE_GEMM_EG
#define MOE_GEMM_EG 2
#endif
#ifndef MOE_GEMM_NPW
#define MOE_GEMM_NPW 1
#endif

// Large batches run on CTA pairs (one MMA of M = 256 over two SMs, each SM holding half of
// the token tile's B rows): per SM, half the activation bytes into shared memory and half
// the operand reads of the MMA.  Four stages (16384 tokens x 128 experts: gate_up 2.00 ms,
// against 2.07 / 2.04 ms with six / seven; one copy-issuing warp, which measured faster than
// two or four).
#ifndef MOE_GEMM_CG
#define MOE_GEMM_CG 2
#endif
#ifndef MOE_GEMM_S2
#define MOE_GEMM_S2 4
#endif
#ifndef MOE_GEMM_S2_FP4
#define MOE_GEMM_S2_FP4 12
#endif
#ifndef MOE_GEMM_NPW2
#define MOE_GEMM_NPW2 1
#endif
#ifndef MOE_GEMM_EG_GU
#define MOE_GEMM_EG_GU MOE_GEMM_EG
#endif

// With MXFP4 activations the packed E2M1 operands take half the shared memory per stage:
// more stages in flight.
#ifndef MOE_GEMV_S_FP4
#define MOE_GEMV_S_FP4 6
#endif
#ifndef MOE_GEMM_S_FP4
#define MOE_GEMM_S_FP4 8
#endif
// MXFP8 activations: a 32-column epilogue read holds 32 tokens (twice the exchange buffer)
#ifndef MOE_GEMM_S_MXFP8
#define MOE_GEMM_S_MXFP8 MOE_GEMM_S
#endif

constexpr int kGemvBN = 8, kGemvNP = MOE_GEMV_NP, kGemvS = MOE_GEMV_S, kGemvCPS = MOE_GEMV_CPS,
              kGemvEG = MOE_GEMV_EG, kGemvNPW = MOE_GEMV_NPW, kGemvDownSplit = MOE_GEMV_DOWN_SPLIT;
constexpr int kGemmBN = 96, kGemmNP = MOE_GEMM_NP, kGemmS = MOE_GEMM_S, kGemmCPS = MOE_GEMM_CPS,
              kGemmEG = MOE_GEMM_EG, kGemmNPW = MOE_GEMM_NPW;
static_assert(kGemvBN >= kMinTileTokens, "tile list sized for the smallest tile");

}  // namespace

// With MXFP8 or MXFP4 activations a token is one MMA column instead of two: tiles of twice
// the tokens keep the same MMA shape.
int expert_tile_tokens(int path, int terms) { return (path == MOE_PATH_GEMV ? kGemvBN : kGemmBN) * (2 / terms); }

int expert_down_split(int path) { return path == MOE_PATH_GEMV ? kGemvDownSplit : 1; }

namespace {
template <int TERMS, bool FP4>
int launch_pair(const FwdArgs& a) {
  constexpr int gv = kGemvBN * 2 / TERMS, gm = kGemmBN * 2 / TERMS;
  constexpr int sv = FP4 ? MOE_GEMV_S_FP4 : kGemvS, sm = FP4 ? MOE_GEMM_S_FP4 : TERMS == 1 ? MOE_GEMM_S_MXFP8 : kGemmS;
  int n1, n2;
  if (a.ws.tile_tokens == gv) {
    n1 = launch_one<MODE_GATE_UP, gv, kGemvNP, sv, kGemvCPS, kGemvEG, kGemvNPW, TERMS, FP4, 1>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, gv, kGemvNP, sv, kGemvCPS, kGemvEG, kGemvNPW, TERMS, FP4, kGemvDownSplit>(a);
  } else if (MOE_GEMM_CG == 2) {
    constexpr int s2 = FP4 ? MOE_GEMM_S2_FP4 : MOE_GEMM_S2;
    n1 = launch_one<MODE_GATE_UP, gm, 1, s2, 1, MOE_GEMM_EG_GU, MOE_GEMM_NPW2, TERMS, FP4, 1, 2>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, gm, 1, s2, 1, kGemmEG, MOE_GEMM_NPW2, TERMS, FP4, 1, 2>(a);
  } else {
    n1 = launch_one<MODE_GATE_UP, gm, kGemmNP, sm, kGemmCPS, kGemmEG, kGemmNPW, TERMS, FP4, 1>(a);
    if (n1 < 0) return -1;
    n2 = launch_one<MODE_DOWN, gm, kGemmNP, sm, kGemmCPS, kGemmEG, kGemmNPW, TERMS, FP4, 1>(a);
  }
  if (n2 < 0) return -1;
  return n1 + n2;
}
}  // namespace

int launch_experts(const FwdArgs& a) {
  if (a.ws.fp4) return launch_pair<1, true>(a);
  return a.ws.terms == 1 ? launch_pair<1, false>(a) : launch_pair<2, false>(a);
}

}  // namespace moe
