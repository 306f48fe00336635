/*
 * moe_mxfp4.h -- C ABI of the B200 (sm_100a) MoE feed-forward layer with MXFP4
 * expert weights (the gpt-oss MoE block).
 *
 * What the layer computes (sources: web pages on gpt-oss, cited by page title
 * and section):
 *   xn   = RMSNorm(x) * norm_w                         ("From GPT-2 to gpt-oss",
 *                                                       sec. 7 RMSNorm; eps from the
 *                                                       llm-atlas GPT-OSS 20B config
 *                                                       table, rms_norm_eps 1e-5)
 *   l    = router_w . xn + router_b   (E logits)      (ewbang.com GPT-OSS article,
 *   top-k experts by logit; w = softmax over the k      section 混合专家模型: a small
 *   selected logits                                     router network picks several
 *                                                       experts and weights them;
 *                                                       top-4 of 32 or 128)
 *   per selected expert e:                             ("From GPT-2 to gpt-oss",
 *     g = W1[e][0:I] . xe,  u = W1[e][I:2I] . xe        sec. 3 Swish/SwiGLU: three
 *     h = silu(min(g, L)) * clamp(u, -L, L)             linears, silu(z)=z*sigmoid(z);
 *     o = W2[e] . h                                     swiglu_limit L = 7 from the
 *                                                       llm-atlas config table)
 *   y    = x + sum_j w_j * o_j                         (ewbang.com article, sections
 *                                                       混合专家模型 and Transformer 块:
 *                                                       weighted mix, block maps
 *                                                       [N x d] to [N x d])
 * Expert weights are MXFP4: 4-bit E2M1 values with one 8-bit E8M0 scale per
 * 32 parameters, 4.25 bits per parameter (ewbang.com article, section
 * 量化 (Quantization)).  xe = bf16(xn); h and y are rounded to bf16.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers unless stated otherwise; the caller
 *     owns and allocates every buffer.  The library allocates and frees no device
 *     memory; besides a per-host-thread launch counter, the per-host-thread CUDA
 *     events of moe_forward_host and the scratch address of moe_forward_no_alloc it
 *     keeps no state between calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on that stream.  The returned status covers the synchronous
 *     argument checks and launch errors only; errors the kernels detect (a
 *     timed-out wait, non-finite input) are recorded in the workspace status
 *     word: read them with moe_device_status().
 *   - No call throws across the ABI or prints.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Device pointers must be 16-byte aligned; MXFP4 code arrays 32-byte aligned.
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null / misaligned pointer, bad size, bad enum */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* block != 32; d or I not a positive multiple of 64;
                                    E not in [1, 256]; top_k not in [1, min(E, 32)];
                                    T*top_k above 2^24 */
  MOE_ERR_WORKSPACE = 3,         /* ws_bytes < moe_workspace_bytes() */
  MOE_ERR_CUDA = 4,              /* a CUDA runtime error at launch */
  MOE_ERR_TIMEOUT = 5,           /* (device) a pipeline wait gave up; the kernel exited cleanly */
  MOE_ERR_NONFINITE = 6,         /* (device) Inf/NaN in the input or the weights */
  MOE_ERR_BOUNDS = 7,            /* (device; bounds-checking builds only, see build.py) a kernel
                                    computed a store address outside its buffer; the store was
                                    skipped */
  MOE_ERR_DEVICE = 8             /* the current device is not sm_100 */
} moe_status;

typedef enum {
  MOE_PATH_AUTO = 0, /* GEMV when tokens per expert are few, else GEMM */
  MOE_PATH_GEMV = 1, /* weight-streaming path: 8-token tiles (16 with MXFP8 activations) */
  MOE_PATH_GEMM = 2  /* grouped GEMM: 96-token tiles (192 with MXFP8 activations) */
} moe_path;

/* Activation format of the expert GEMMs (the weights are MXFP4 in both).
 * MOE_ACT_BF16: the expert inputs xe = bf16(RMSNorm(x)) and the SwiGLU outputs h are used
 *   exactly as bf16 (each carried to the tensor cores as two E4M3 terms with their block
 *   scales; exact for every value above 2^-13 of its 32-block's largest).  The layer as the
 *   pages state it.
 * MOE_ACT_MXFP8: xe and h are quantized to MXFP8 before each projection: in 32-value blocks
 *   along the projection's reduction axis (the pages' block of one 8-bit scale per 32
 *   values), scale 2^(floor(log2 amax) - 7) clamped to [2^-122, 2^126] (1 for an all-zero
 *   block), elements rounded to the nearest OCP FP8 E4M3 value (ties to even).  Half the
 *   activation bytes and tensor-core work; the E4M3 rounding moves the expert output
 *   (y - x) by about 5% of its norm at gpt-oss width, more than the exact layer's parity
 *   tolerance on y.  An extension: the pages quantize only the weights.
 * MOE_ACT_MXFP4: xe and h are quantized to MXFP4, the expert weights' own format and rule
 *   (E2M1 elements, one E8M0 scale per 32 values along the projection's reduction axis,
 *   scale 2^(floor(log2 amax) - 2) clamped to [2^-127, 2^127], elements rounded to the
 *   nearest E2M1 value, ties to even, saturating at 6).  The expert GEMMs then run the
 *   FP4 x FP4 block-scaled MMA (the FP4 rate) on the weight codes as stored; a quarter of
 *   the bf16 activation bytes.  The E2M1 rounding moves the expert output far more than
 *   MXFP8's (about 22% of y - x at gpt-oss width, against MXFP8's 5%); also an
 *   extension. */
typedef enum {
  MOE_ACT_BF16 = 0,
  MOE_ACT_MXFP8 = 1,
  MOE_ACT_MXFP4 = 2
} moe_act_format;

/* Which projection a weight tensor is (sets its row order in storage). */
typedef enum {
  MOE_WEIGHT_PLAIN = 0,   /* any [E][N][K], rows stored in order (W2, the down projection) */
  MOE_WEIGHT_GATE_UP = 1  /* W1 [E][2I][d]: gate rows 0..I-1, up rows I..2I-1 */
} moe_weight_role;

typedef struct {
  int32_t d;            /* hidden size (gpt-oss: 2880)                                  */
  int32_t I;            /* expert intermediate size (gpt-oss: 2880)                     */
  int32_t E;            /* experts (gpt-oss-20b: 32, gpt-oss-120b: 128)                 */
  int32_t top_k;        /* experts per token (gpt-oss: 4)                               */
  int32_t block;        /* MXFP4 block size; must be 32                                 */
  float rms_eps;        /* RMSNorm epsilon (gpt-oss: 1e-5)                              */
  float swiglu_limit;   /* SwiGLU clamp (gpt-oss: 7)                                    */
  int32_t path;         /* a moe_path value                                             */
  int32_t act_format;   /* a moe_act_format value: the expert GEMMs' activation format  */
} moe_dims;

/* ---------------------------------------------------------------- MXFP4 storage
 * A weight tensor [E][N][K] (K = reduction axis, a multiple of 64; N a multiple of 64)
 * is stored in the form the tensor cores' block-scaled MMA reads, in tiles of 128 rows
 * x 128 k.  With NT = ceil(N/128) and KC = ceil(K/128):
 *   codes  [E][NT][KC][128][64] bytes: one contiguous 8 KB block per tile; byte j of
 *          row r of block [e][t][c] holds the E2M1 codes of row 128t + r at
 *          k = 128c + 2j (low nibble) and k = 128c + 2j + 1 (high nibble); codes of
 *          rows >= N or k >= K are 0.  Code bits: sign (bit 3), exponent (bits 2..1,
 *          bias 1), mantissa (bit 0).
 *   scales [E][NT][KC][512] bytes: the E8M0 scale 2^(byte - 127) of (row n, 32-value
 *          block b) is byte (n%32)*16 + ((n%128)/32)*4 + b%4 of the 512-byte group
 *          [e][n/128][b/4] (the tensor cores' scale-factor layout: 128 rows x 4
 *          blocks); bytes of rows >= N or blocks >= K/32 are 127.
 * For MOE_WEIGHT_GATE_UP the rows are stored in the order of 128-row tiles that each
 * pair 64 gate rows with the 64 matching up rows: stored row 128*t + r holds gate row
 * 64*t + r (r < 64) or up row I + 64*t + r - 64 (r >= 64); I must be a multiple of 64.
 * Payload: 4.25 bits per parameter (plus the zero padding up to 128 rows and 128 k).
 */
size_t moe_mxfp4_codes_bytes(int32_t E, int32_t N, int32_t K);  /* E*NT*KC*8192 */
size_t moe_mxfp4_scales_bytes(int32_t E, int32_t N, int32_t K); /* E*NT*KC*512 */

/* Quantize fp32 weights w [E][N][K] (device, row-major) to MXFP4 (codes, scales as above).
 * Per 32-value block: s = clamp(floor(log2(amax)) - 2, -127, 127); each value
 * x * 2^-s is rounded to the nearest E2M1 value (ties to the even code), saturating
 * at +-6; the sign bit is set only on non-zero codes; an all-zero block gets s = 0.
 * (ewbang.com article, section 量化: 4-bit values, one 8-bit scale per 32.)
 * role: a moe_weight_role (MOE_WEIGHT_GATE_UP needs N = 2I with I a multiple of 64).
 * status_word: optional device int32; MOE_ERR_NONFINITE is OR-ed into it when a
 * block holds Inf/NaN (that block's scale byte is then 0xFF, the E8M0 NaN).
 * Errors: MOE_ERR_INVALID_ARG (null/misaligned pointer, E/N/K <= 0, bad role),
 * MOE_ERR_UNSUPPORTED_SHAPE (N or K not a multiple of 64; GATE_UP with N/2 not a
 * multiple of 64), MOE_ERR_CUDA. */
moe_status moe_mxfp4_quantize(const float* w, int32_t E, int32_t N, int32_t K, int32_t role, uint8_t* codes,
                              uint8_t* scales, int32_t* status_word, void* stream);

/* Bytes of device scratch moe_route / moe_forward need for T tokens.  The first 256
 * bytes hold the device status word; the rest is scratch that the calls overwrite.
 * Calls that share a workspace must be ordered on one stream. */
size_t moe_workspace_bytes(const moe_dims* dims, int32_t T);

/* Steps 1-4 of the layer for T tokens: RMSNorm, router logits, top-k + softmax, and
 * token-to-expert grouping.
 *   x        [T][d] bf16          norm_w [d] fp32        router_w [E][d] fp32
 *   router_b [E] fp32 or NULL (zero bias)
 * Outputs (device; each may be NULL except as noted):
 *   topk_idx [T][k] int32  expert ids, by logit descending (ties: lower id first)
 *   topk_w   [T][k] fp32   softmax over the k selected logits (sums to 1 per token)
 *   counts   [E]    int32  tokens routed to each expert (sum = T*k)
 *   offsets  [E+1]  int32  exclusive prefix sum of counts
 *   perm     [T*k]  int32  pair list sorted by (expert asc, token asc); entry = t*k + slot
 * The router runs in fp32 on the unrounded RMSNorm output.
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_WORKSPACE, MOE_ERR_CUDA;
 * device side: MOE_ERR_NONFINITE (non-finite logits). */
moe_status moe_route(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                     const float* router_w, const float* router_b, int32_t* topk_idx, float* topk_w,
                     int32_t* counts, int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes,
                     void* stream);

/* The whole layer: y [T][d] bf16 = x + MoE(RMSNorm(x)).
 *   w1_codes / w1_scales: W1 [E][2I][d] in the MXFP4 storage above, role GATE_UP
 *   w2_codes / w2_scales: W2 [E][d][I], role PLAIN
 * Optional outputs (device, NULL to skip): topk_idx_out [T][k], topk_w_out [T][k],
 * counts_out [E].
 * y may not alias x.  T >= 1 (T = 0 returns MOE_OK and launches nothing).
 * Arithmetic: the expert projections run on the tensor cores' block-scaled MMA
 * (E2M1 weights with their E8M0 scales, as stored) with fp32 accumulation.  With
 * MOE_ACT_BF16 each activation (xe, then h) enters as two E4M3 terms with one E8M0 scale
 * per 32 values each: hi = RN(v / 2^s1), lo = RN((v - hi * 2^s1) / 2^s2), s1 and s2 set by
 * the largest |v| and the largest residual of the block.  hi + lo equals v whenever
 * |v| >= 2^-13 * max|block|; smaller values are off by at most 2^-20 * max|block|.  With
 * MOE_ACT_MXFP8 the hi term alone enters, with MOE_ACT_MXFP4 E2M1 codes (FP4 x FP4 MMA; see
 * moe_act_format).  The k routing-weighted expert outputs stay fp32 and are added to the
 * residual in a fixed order (slot, then reduction-axis split): results do not depend on
 * scheduling, and repeated calls give identical y.
 * Errors: as moe_route. */
moe_status moe_forward(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                       const float* router_w, const float* router_b, const uint8_t* w1_codes,
                       const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                       uint16_t* y, int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out,
                       void* ws, size_t ws_bytes, void* stream);

/* moe_forward plus per-kernel timing: `events` is an array of n_events cudaEvent_t
 * handles created by the caller (timing enabled).  Event 2i is recorded on `stream`
 * just before the i-th kernel this call launches and event 2i+1 just after it, until
 * the array runs out.  Recording adds no synchronization; when `stream` is being captured
 * into a CUDA graph the events are recorded as external event nodes of the graph, so
 * that every replay records them.  The kernels of a call are, in order: route
 * (RMSNorm + router + top-k + E4M3 split of xe), group, pack (the token tiles' packed
 * activation blocks), gate_up, down, combine; on the GEMV path with T <= 64, route (which
 * then also groups), pack, gate_up, down and combine.
 * Errors: as moe_forward; MOE_ERR_INVALID_ARG if n_events < 0 or events is NULL with
 * n_events > 0. */
moe_status moe_forward_timed(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                             const float* router_w, const float* router_b, const uint8_t* w1_codes,
                             const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                             uint16_t* y, int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out,
                             void* ws, size_t ws_bytes, void* stream, void* const* events, int32_t n_events);

/* moe_forward, and in the same pass the next block's first RMSNorm of the output
 * (every block holds two RMSNorms and maps [N x d] to [N x d]: ewbang.com article, section
 * Transformer 块):
 *   y      [T][d] bf16 = x + MoE(RMSNorm(x))                    (as moe_forward)
 *   y_norm [T][d] bf16 = bf16(y / sqrt(mean(y^2) + next_eps) * next_norm_w), on the bf16 y
 * next_norm_w [d] fp32 (device), next_eps >= 0.  The routing-weighted sum of the k expert
 * outputs, the residual add and the RMSNorm run in one pass over each token's row (on
 * both paths; the small-batch path then does not fold the sum into the down GEMM).
 * y and y_norm may not alias x or each other.  Errors: as moe_forward; MOE_ERR_INVALID_ARG
 * for a null / misaligned next_norm_w or y_norm, or a negative or non-finite next_eps. */
moe_status moe_forward_norm(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                            const float* router_w, const float* router_b, const uint8_t* w1_codes,
                            const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                            const float* next_norm_w, float next_eps, uint16_t* y, uint16_t* y_norm, void* ws,
                            size_t ws_bytes, void* stream);

/* One slice of the intermediate features, for splitting a layer over G GPUs (tensor
 * parallelism over I; the pages run the layer on one GPU, this is an extension).  The
 * expert MLP is separable over its intermediate features: h's feature i depends only on
 * W1's gate row i and up row I + i, and the down projection sums W2[:, i] * h_i over i.
 * A rank holds, for every expert, the gate rows [i0, i1) and up rows [I + i0, I + i1) of
 * W1 and the columns [i0, i1) of W2, quantized as the layer of intermediate size
 * dims->I = i1 - i0 (a multiple of 64; W1 with role MOE_WEIGHT_GATE_UP, W2 plain; since i0
 * is a multiple of 64 the slice's MXFP4 blocks are those of the whole matrix).  Every rank
 * routes the same x with the same router and gets the same experts.  The call writes
 *   y_partial [T][d] fp32 = sum_j w_j * W2[e_j][:, i0:i1] . h_j[i0:i1]   (no residual)
 * The sum of y_partial over slices that cover [0, I) (one all-reduce) is the expert mix of
 * the whole layer; moe_residual_norm then gives y = bf16(x + sum).
 * y_partial may not alias x.  Errors: as moe_forward. */
moe_status moe_forward_partial(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                               const float* router_w, const float* router_b, const uint8_t* w1_codes,
                               const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                               float* y_partial, int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out,
                               void* ws, size_t ws_bytes, void* stream);

/* y [T][d] bf16 = bf16(x + s) for s [T][d] fp32 (device; e.g. the all-reduced outputs of
 * moe_forward_partial), and with norm_w non-NULL also the next block's RMSNorm
 * y_norm = bf16(y / sqrt(mean(y^2) + eps) * norm_w) on the bf16 y.  One launch.
 * d a positive multiple of 64; y and y_norm may not alias x or each other.
 * Errors: MOE_ERR_INVALID_ARG (T < 0, d <= 0, null / misaligned pointer, bad eps),
 * MOE_ERR_UNSUPPORTED_SHAPE (d not a multiple of 64), MOE_ERR_DEVICE, MOE_ERR_CUDA. */
moe_status moe_residual_norm(int32_t T, int32_t d, const uint16_t* x, const float* s, const float* norm_w,
                             float eps, uint16_t* y, uint16_t* y_norm, void* stream);

/* moe_forward from host memory to host memory, with the copies overlapped with the layer.
 *   x_host, y_host [T][d] bf16, host memory, page-locked (cudaHostAlloc / cudaHostRegister)
 *                  for the copies to overlap, and required when `stream` is being captured
 *   x_dev, y_dev   [T][d] bf16, device buffers the call stages through (distinct)
 * The other arguments are moe_forward's (device pointers).  The T tokens run as consecutive
 * chunks of chunk_tokens tokens (the last one shorter; 0 = the library's choice, which
 * moe_host_chunk_tokens returns).  With one chunk the copy in, the layer and the copy out
 * run in order on `stream`.  With several, chunk c is copied in on h2d_stream, its layer
 * runs on `stream` and it is copied out on d2h_stream, so that the copies of the chunks
 * before and after it overlap its layer (PCIe carries both directions at once); the copies
 * in first wait for the work enqueued on `stream` before the call, and `stream` waits for
 * the last copy out at the end.  NULL h2d_stream / d2h_stream: those copies run on
 * `stream` too.  The call returns once everything is enqueued; y_host is complete when
 * `stream` has passed the call (the caller synchronizes).  A token's routing and expert
 * outputs do not depend on the other tokens of its batch, so y_host is moe_forward's y of
 * each chunk; the down GEMM's split of its reduction axis follows the chunk's tile count,
 * so y may differ in the last bf16 bit from a single moe_forward over all T tokens (both
 * follow the layer's definition within the same bound).  ws: moe_workspace_bytes(dims,
 * chunk) bytes at least (and for the last chunk's size), reused chunk after chunk.
 * The kernels count as in moe_forward, summed over the chunks.  Everything is enqueued
 * per chunk on the caller's streams; the call allocates nothing on the device.
 * Errors: as moe_forward, checked before anything is enqueued; MOE_ERR_INVALID_ARG for
 * chunk_tokens < 0 or a null / misaligned / aliased x_dev or y_dev; MOE_ERR_WORKSPACE when
 * ws is smaller than a chunk needs. */
moe_status moe_forward_host(const moe_dims* dims, int32_t T, const uint16_t* x_host, uint16_t* y_host,
                            uint16_t* x_dev, uint16_t* y_dev, const float* norm_w, const float* router_w,
                            const float* router_b, const uint8_t* w1_codes, const uint8_t* w1_scales,
                            const uint8_t* w2_codes, const uint8_t* w2_scales, void* ws, size_t ws_bytes,
                            int32_t chunk_tokens, void* stream, void* h2d_stream, void* d2h_stream);

/* Tokens per chunk that moe_forward_host takes for chunk_tokens = 0: all T (one chunk) on
 * the small-batch path and below 4096 tokens, else ceil(T / n) for n = min(4, T / 2048)
 * chunks.  Returns -1 for invalid dims. */
int32_t moe_host_chunk_tokens(const moe_dims* dims, int32_t T);

/* The path moe_forward takes for these dims and T: dims->path, or for MOE_PATH_AUTO the
 * choice it makes (MOE_PATH_GEMV when T*top_k/E <= 24 tokens per expert, else
 * MOE_PATH_GEMM).  Returns -1 for invalid dims. */
int32_t moe_resolve_path(const moe_dims* dims, int32_t T);

/* Byte offsets of the workspace's sub-buffers for T tokens, for inspection by tests and
 * debuggers (layout may change between versions).  offsets[0..MOE_WS_FIELDS-2] receive,
 * in order: status, counts (int32 [E], then internal counters), offsets, ntiles,
 * tile_base (int32 [E]: first token tile of each expert), tiles, topk_idx, topk_w, perm,
 * inv, w_sorted,
 * xq  [T][2][dp] E4M3 (hi and lo terms of xe = bf16(xn) per token; dp = d rounded up to
 *     a multiple of 128), xsf [T][2][dp/32] E8M0 (their scales),
 * bpx / bph: packed activation blocks of xe and of the SwiGLU output h, per token tile
 *     and 128-chunk: the tile's 2 * BN E4M3 rows (hi / lo term of each token; BN = 8 on
 *     the GEMV path, 96 on the GEMM path) or, with MOE_ACT_MXFP8, its BN rows (one per
 *     token; BN = 16 / 192), in the tensor cores' 128-byte-swizzled order, then their
 *     scales,
 * ys  [S][T*k][d] fp32 (weighted expert outputs, row t*k + slot; S = 6 planes of partial sums
 *     on the GEMV path, whose down GEMM splits its reduction axis in up to six, else 1);
 * offsets[MOE_WS_FIELDS-1] = total bytes.  Errors: MOE_ERR_INVALID_ARG,
 * MOE_ERR_UNSUPPORTED_SHAPE. */
#define MOE_WS_FIELDS 17
moe_status moe_workspace_layout(const moe_dims* dims, int32_t T, size_t* offsets);

/* Synchronize `stream`, then read and clear the device status word of workspace `ws`
 * (device pointer).  Returns MOE_OK or the first device-side error recorded since the
 * last read (MOE_ERR_TIMEOUT, MOE_ERR_NONFINITE), or MOE_ERR_CUDA. */
moe_status moe_device_status(void* ws, void* stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status status);

/* Number of kernels the last successful moe_forward / moe_route call on this host
 * thread launched (for launch accounting in benchmarks). */
int32_t moe_last_launch_count(void);

/* moe_forward for callers that cannot allocate device memory: it takes no workspace and
 * allocates nothing (no cudaMalloc, no library allocator).  The pages have no
 * counterpart; this is a deployment convenience.  Callers that run where allocation is
 * not available -- inside an allocator or memory-pool callback, in a plugin host that
 * lends out only its own tensors, or in a serving loop that forbids cudaMalloc and its
 * implicit synchronization once it is running -- use it instead of moe_forward.
 * Scratch: a fixed 16 MiB array in the library's own device memory, present on every GPU
 * that loads the library until the process exits.  T whose moe_workspace_bytes() exceed
 * 16 MiB is rejected with MOE_ERR_WORKSPACE (at d = I = 2880, E = 32, top-4: up to 34
 * tokens).
 * The first call in a CUDA context (normally a device's primary context) looks up the
 * array's device address in that context (cudaGetSymbolAddress) and remembers it for that
 * context; make that first call before any stream capture.  After cudaDeviceReset the
 * next call in the new context looks the address up again.
 * All calls share the one array and it keeps the previous call's contents; the device
 * status word and the expert counters are cleared by every call.  Calls that overlap on
 * the GPU (unordered streams, or several host threads) race on the array.
 * Arguments as moe_forward; status_out (device int32, 4-byte aligned, may be NULL)
 * receives the call's device status word (0 = MOE_OK) on `stream` once the call's kernels
 * have run (with T = 0: 0).  When the call returns an error, status_out is not written.
 * Errors: as moe_forward (the same codes for the same argument errors), and
 * MOE_ERR_WORKSPACE for T beyond the array. */
moe_status moe_forward_no_alloc(const moe_dims* dims, int32_t T, const uint16_t* x, const float* norm_w,
                                const float* router_w, const float* router_b, const uint8_t* w1_codes,
                                const uint8_t* w1_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                                uint16_t* y, int32_t* status_out, void* stream);

/* Test hook for the device-side failure path.  With enable != 0, the next moe_forward
 * (or moe_forward_timed) call on this host thread launches its gate_up kernel with one pipeline arrival withheld in its first CTA: that CTA's bounded
 * wait expires after about 2 s, the CTA drains its copies, frees its tensor memory and
 * exits, and the workspace status word records MOE_ERR_TIMEOUT (y of that call is then
 * unspecified).  The hook clears itself after that call; nothing faults or hangs. */
void moe_debug_inject_timeout(int32_t enable);

#ifdef __cplusplus
}
#endif

#endif /* MOE_MXFP4_H */
