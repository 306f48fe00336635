// CPU oracle of the gpt-oss MoE feed-forward layer with MXFP4 expert weights.
//
// TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
// CPU-baseline leg may load this library.  The product path never calls it and
// shares no code with it (no headers, tables or helpers in common).
//
// Plain, slow, obviously correct: fp64 arithmetic, one accumulator per dot
// product, the MXFP4 code table written out, no blocking or reordering.
// Activations are rounded to bfloat16 exactly where the layer stores bf16:
// the expert input xe = bf16(RMSNorm(x)), the SwiGLU output h, and the output y.
//
// Sources (web pages on gpt-oss; cited by page and section):
//  [R-zh]   "從GPT-2到gpt-oss" (新智元 translation of S. Raschka,
//           "From GPT-2 to gpt-oss: Analyzing the Architectural Advances"):
//           sec. 3 (Swish = x*sigmoid(x); GLU/SwiGLU with three linears; the
//           width-1024 parameter-count example), sec. 4 (MoE replaces the single
//           FFN; only a subset of experts active per token), sec. 7 (RMSNorm
//           divides by the RMS, no mean subtraction, no bias), "MXFP4優化"
//           (MoE experts shipped in MXFP4).
//  [ARCH]   ewbang.com article on the GPT-OSS architecture: "Transformer 块"
//           (two RMSNorms per block; block input/output [N x 2880]),
//           "混合专家模型（MoE）" (router picks several experts per token and
//           weights them, e.g. 0.7*NN2 + 0.3*NN4; top-4 of 32 or 128),
//           "量化（Quantization）" (4-bit values, one 8-bit scale per 32
//           parameters, 4.25 bits per parameter).
//  [ATLAS]  llm-atlas "GPT-OSS 20B" model page, raw config table:
//           hidden_size 2880, intermediate_size 2880, num_local_experts 32/128,
//           experts_per_token 4, hidden_act silu, rms_norm_eps 1e-5,
//           swiglu_limit 7.
//
// Readings where the pages are silent (each listed with its reason in the
// design notes of the repository):
//  * MXFP4 element = E2M1 (the pages say "4-bit float"); scale = E8M0 power of
//    two 2^(byte-127); the 32-element block runs along K (the reduction axis) of
//    each weight row; scale exponent s = floor(log2(amax)) - 2, clamped to
//    [-127, 127]; elements x*2^-s rounded to nearest E2M1 value, ties to the
//    even code, saturating at +-6; an all-zero block gets byte 127.
//  * Router: logits = b + W_r * xn on the unrounded (fp64 here) RMSNorm output;
//    top-k by (logit descending, index ascending); weights = softmax over the k
//    selected logits.
//  * SwiGLU clamp (swiglu_limit 7): h = silu(min(g, 7)) * clamp(u, -7, 7);
//    W1 rows 0..I-1 are the gate, rows I..2I-1 the up projection.
//  * Block: y = x + sum_j w_j * Expert_j(bf16(RMSNorm(x))), j in slot order.
//  * Optional MXFP8 activations (act_format 1; the pages quantize only the expert
//    weights, so this mode is an extension): the expert inputs xe and the SwiGLU
//    outputs h are each cut into 32-value blocks along the expert's reduction
//    axis, the block structure [ARCH] "量化" gives for the weights, with an 8-bit
//    element: OCP FP8 E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits;
//    subnormals below 2^-6; largest finite 448; the pattern with all exponent
//    and mantissa bits set is NaN).  Block scale X = 2^s, s = floor(log2(amax))
//    - 7 (amax / X lands in [128, 256)), clamped to [-122, 126], s = 0 for an
//    all-zero block; element = X * (E4M3 value nearest to v / X, ties to the
//    even code, saturating at 448).
//  * Optional MXFP4 activations (act_format 2; also an extension): the same points and
//    blocks, with the expert weights' own format ([ARCH] "量化": 4-bit values, one
//    8-bit scale per 32): E2M1 elements and the weights' scale rule, s = floor(log2
//    amax) - 2 clamped to [-127, 127] (s = 0 for an all-zero block), element =
//    2^s * (E2M1 value nearest to v / 2^s, ties to the even code, saturating at 6).
//
// Oracle storage layout (its own, documented here): codes [rows][K/2], two codes
// per byte, low nibble = even k; scale bytes [rows][K/32].
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// E2M1 magnitudes by the 3 low bits of a code: exponent bits e1 e0, mantissa m.
// e = 0 is subnormal (0 or 0.5); otherwise 2^(e-1) * (1 + m/2).
const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double e2m1_value(int code) {
  const double mag = kE2M1[code & 7];
  return (code & 8) ? -mag : mag;
}

// bfloat16 <-> double.  bf16 keeps 8 significant bits and float's exponent
// range; rounding is to nearest, ties to even, directly from the double.
double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

double round_to_bf16(double v) {
  if (v == 0.0 || !std::isfinite(v)) return v;
  const double a = std::fabs(v);
  double r;
  if (a < 0x1.0p-126) {
    // subnormal range: fixed quantum 2^-133
    r = std::nearbyint(a * 0x1.0p133) * 0x1.0p-133;
  } else {
    int e;
    const double m = std::frexp(a, &e);             // a = m * 2^e, m in [0.5, 1)
    r = std::ldexp(std::nearbyint(std::ldexp(m, 8)), e - 8);  // 8 significant bits
    if (r > 0x1.FEp127) r = std::numeric_limits<double>::infinity();
  }
  return v < 0 ? -r : r;
}

uint16_t bf16_bits_of(double v_rounded) {
  const float f = (float)v_rounded;  // exact: v_rounded is a bf16 value
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

// floor(log2(a)) for finite a > 0, from the exponent alone (exact, unlike log2).
int floor_log2(double a) {
  int e;
  std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1)  =>  floor(log2 a) = e - 1
  return e - 1;
}

// Nearest E2M1 code to |v| (v already divided by the block scale), ties to the
// even code, saturating at 6.  Written as "closest grid point" so that it does
// not depend on threshold tables.
int nearest_e2m1_magnitude_code(double a) {
  if (a >= 6.0) return 7;
  int best = 0;
  double best_err = std::fabs(a - kE2M1[0]);
  for (int c = 1; c < 8; ++c) {
    const double err = std::fabs(a - kE2M1[c]);
    if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) != 0)) {
      best = c;
      best_err = err;
    }
  }
  return best;
}

// The finite non-negative E4M3 values in code order (codes 0x00..0x7E), from the
// format's fields: exponent field e (bits 6..3, bias 7), mantissa m (bits 2..0);
// e = 0 is subnormal, m/8 * 2^-6; otherwise (1 + m/8) * 2^(e-7).  0x7F is NaN.
const std::vector<double>& e4m3_grid() {
  static const std::vector<double> grid = [] {
    std::vector<double> g;
    for (int code = 0; code < 0x7F; ++code) {
      const int e = code >> 3, m = code & 7;
      g.push_back(e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7));
    }
    return g;
  }();
  return grid;
}

// Nearest E4M3 magnitude to a >= 0, ties to the even code, saturating at 448.
int nearest_e4m3_code(double a) {
  const std::vector<double>& g = e4m3_grid();
  if (!(a > 0.0)) return 0;
  if (a >= g.back()) return (int)g.size() - 1;
  const int hi = (int)(std::lower_bound(g.begin(), g.end(), a) - g.begin());   // g[hi] >= a > g[hi-1]
  const int lo = hi - 1;
  const double dlo = a - g[lo], dhi = g[hi] - a;
  if (dlo < dhi) return lo;
  if (dhi < dlo) return hi;
  return (lo & 1) ? hi : lo;
}

// MXFP8 quantization of one block of n <= 32 values in place (see the header).
void mxfp8_block(double* v, int n, int32_t* exp_out) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  const int s = amax > 0.0 ? std::min(126, std::max(-122, floor_log2(amax) - 7)) : 0;
  for (int i = 0; i < n; ++i) {
    const double q = e4m3_grid()[nearest_e4m3_code(std::ldexp(std::fabs(v[i]), -s))];
    v[i] = std::copysign(std::ldexp(q, s), v[i]);
    if (q == 0.0) v[i] = 0.0;
  }
  if (exp_out) *exp_out = s;
}

// MXFP4 quantization of one block of n <= 32 values in place, by the rule the expert
// weights are quantized with (oracle_quantize): 2^s * nearest E2M1 value of v / 2^s.
void mxfp4_block(double* v, int n) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  const int s = amax > 0.0 ? std::clamp(floor_log2(amax) - 2, -127, 127) : 0;
  for (int i = 0; i < n; ++i) {
    const int c = nearest_e2m1_magnitude_code(std::fabs(std::ldexp(v[i], -s)));
    v[i] = c == 0 ? 0.0 : std::copysign(std::ldexp(kE2M1[c], s), v[i]);
  }
}

// The activation format's quantization of one 32-block (act_format 1: MXFP8, 2: MXFP4).
void quantize_activation_block(double* v, int32_t act_format) {
  if (act_format == 1) mxfp8_block(v, 32, nullptr);
  else if (act_format == 2) mxfp4_block(v, 32);
}

template <class F>
void parallel_chunks(int64_t n, int nthreads, F&& body) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  nthreads = (int)std::min<int64_t>(nthreads, std::max<int64_t>(1, n));
  if (nthreads == 1) {
    body(0, n);
    return;
  }
  std::vector<std::thread> ts;
  const int64_t chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    const int64_t b = (int64_t)t * chunk, e = std::min(n, b + chunk);
    if (b >= e) break;
    ts.emplace_back([&body, b, e] { body(b, e); });
  }
  for (auto& t : ts) t.join();
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// MXFP4 storage ([ARCH] 量化: 4-bit value + one 8-bit scale per 32 params).
// ---------------------------------------------------------------------------

int64_t oracle_mxfp4_code_bytes(int64_t rows, int32_t K) { return rows * (K / 2); }
int64_t oracle_mxfp4_scale_bytes(int64_t rows, int32_t K) { return rows * (K / 32); }

double oracle_e2m1_value(int32_t code) { return e2m1_value(code & 15); }

// Quantize fp32 rows [rows][K] (K % 32 == 0).  Returns 0, or 1 if any input is
// not finite (outputs for such blocks are unspecified).
int32_t oracle_quantize(const float* w, int64_t rows, int32_t K, uint8_t* codes, uint8_t* scales) {
  if (K % 32 != 0) return 2;
  const int nb = K / 32;
  std::atomic<int32_t> any_bad{0};
  // Rows are independent; split them over threads.
  parallel_chunks(rows, 0, [&](int64_t r0, int64_t r1) {
  int32_t status = 0;
  for (int64_t r = r0; r < r1; ++r) {
    for (int b = 0; b < nb; ++b) {
      const float* blk = w + r * K + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) {
        const double v = (double)blk[i];
        if (!std::isfinite(v)) status = 1;
        amax = std::max(amax, std::fabs(v));
      }
      int s = 0;  // all-zero block: scale 2^0
      if (amax > 0.0 && std::isfinite(amax)) s = std::clamp(floor_log2(amax) - 2, -127, 127);
      scales[r * nb + b] = (uint8_t)(s + 127);
      for (int i = 0; i < 32; ++i) {
        const double v = std::ldexp((double)blk[i], -s);   // exact power-of-two scaling
        int c = nearest_e2m1_magnitude_code(std::fabs(v));
        if (v < 0 && c != 0) c |= 8;                         // sign only on non-zero codes
        const int64_t k = (int64_t)b * 32 + i;
        uint8_t& byte = codes[r * (K / 2) + k / 2];
        if ((k & 1) == 0) byte = (uint8_t)((byte & 0xF0) | c);
        else byte = (uint8_t)((byte & 0x0F) | (c << 4));
      }
    }
  }
  if (status) any_bad = 1;
  });
  return any_bad.load();
}

// Decode rows to fp64: value = E2M1(code) * 2^(byte - 127).  Returns 1 if a
// scale byte is 0xFF (the E8M0 NaN encoding), else 0.
int32_t oracle_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int32_t K, double* out) {
  std::atomic<int32_t> status{0};
  const int nb = K / 32;
  // Every element is decoded on its own; rows are split over threads.
  parallel_chunks(rows, 0, [&](int64_t r0, int64_t r1) {
    for (int64_t r = r0; r < r1; ++r)
      for (int32_t k = 0; k < K; ++k) {
        const uint8_t byte = codes[r * (K / 2) + k / 2];
        const int c = (k & 1) ? (byte >> 4) : (byte & 15);
        const uint8_t sb = scales[r * nb + k / 32];
        if (sb == 0xFF) status = 1;
        out[r * K + k] = e2m1_value(c) * std::ldexp(1.0, (int)sb - 127);
      }
  });
  return status.load();
}

// ---------------------------------------------------------------------------
// bf16 helpers exposed for the oracle's own pins.
// ---------------------------------------------------------------------------
double oracle_round_bf16(double v) { return round_to_bf16(v); }

// bf16 bit patterns of n doubles, each rounded to nearest (ties to even) as above.
void oracle_to_bf16(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_of(round_to_bf16(v[i]));
}

// E4M3 code (0..0x7E) of the value nearest to |a|, ties to the even code, saturating.
int32_t oracle_e4m3_nearest_code(double a) { return nearest_e4m3_code(std::fabs(a)); }
double oracle_e4m3_value(int32_t code) { return (code >= 0 && code < 0x7F) ? e4m3_grid()[code] : NAN; }

// MXFP4 quantization (the weights' rule) of n values (n a multiple of 32) in 32-value
// blocks.  Returns 0, or 2 if n % 32 != 0.
int32_t oracle_mxfp4_quantize_values(const double* v, int64_t n, double* out) {
  if (n % 32) return 2;
  for (int64_t b = 0; b < n / 32; ++b) {
    std::memcpy(out + 32 * b, v + 32 * b, 32 * sizeof(double));
    mxfp4_block(out + 32 * b, 32);
  }
  return 0;
}

// MXFP8 quantization of n values (n a multiple of 32) in 32-value blocks; exps[n/32]
// receives the block scale exponents (nullable).  Returns 0, or 2 if n % 32 != 0.
int32_t oracle_mxfp8_quantize(const double* v, int64_t n, double* out, int32_t* exps) {
  if (n % 32) return 2;
  for (int64_t b = 0; b < n / 32; ++b) {
    std::memcpy(out + 32 * b, v + 32 * b, 32 * sizeof(double));
    mxfp8_block(out + 32 * b, 32, exps ? exps + b : nullptr);
  }
  return 0;
}

// ---------------------------------------------------------------------------
// RMSNorm ([R-zh] sec. 7; eps = rms_norm_eps from [ATLAS]):
//   xn_i = x_i / sqrt(mean_j x_j^2 + eps) * gamma_i
// ---------------------------------------------------------------------------
void oracle_rmsnorm(int32_t T, int32_t d, const uint16_t* x, const float* gamma, double eps, double* xn) {
  for (int32_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      const double v = bf16_bits_to_double(x[(int64_t)t * d + i]);
      ss += v * v;
    }
    const double r = 1.0 / std::sqrt(ss / d + eps);
    for (int32_t i = 0; i < d; ++i)
      xn[(int64_t)t * d + i] = bf16_bits_to_double(x[(int64_t)t * d + i]) * r * (double)gamma[i];
  }
}

// ---------------------------------------------------------------------------
// Router ([ARCH] 混合专家模型: a small network scores the experts; top-k of
// E; the chosen experts are mixed with weights).  For each token:
//   l_e = b_e + sum_i W_r[e,i] * xn_i       (xn unrounded)
//   top-k by (l desc, e asc); w = softmax over the k selected logits
//   gap = l_(k) - l_(k+1)  (+inf when k == E)
// Outputs: idx [T][k], w [T][k]; logits [T][E] and gap [T] are optional.
// ---------------------------------------------------------------------------
void oracle_route(int32_t T, int32_t d, int32_t E, int32_t k, const uint16_t* x, const float* gamma,
                  double eps, const float* router_w, const float* router_b, int32_t* idx, double* w,
                  double* logits_out, double* gap_out, int32_t nthreads) {
  parallel_chunks(T, nthreads, [&](int64_t t0, int64_t t1) {
    std::vector<double> xn(d), l(E);
    std::vector<int32_t> order(E);
    for (int64_t t = t0; t < t1; ++t) {
      oracle_rmsnorm(1, d, x + t * d, gamma, eps, xn.data());
      for (int32_t e = 0; e < E; ++e) {
        double acc = router_b ? (double)router_b[e] : 0.0;
        for (int32_t i = 0; i < d; ++i) acc += (double)router_w[(int64_t)e * d + i] * xn[i];
        l[e] = acc;
      }
      for (int32_t e = 0; e < E; ++e) order[e] = e;
      std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
        return l[a] > l[b] || (l[a] == l[b] && a < b);
      });
      const double lmax = l[order[0]];
      double z = 0.0;
      for (int32_t j = 0; j < k; ++j) z += std::exp(l[order[j]] - lmax);
      for (int32_t j = 0; j < k; ++j) {
        idx[t * k + j] = order[j];
        w[t * k + j] = std::exp(l[order[j]] - lmax) / z;
      }
      if (logits_out)
        for (int32_t e = 0; e < E; ++e) logits_out[t * E + e] = l[e];
      if (gap_out)
        gap_out[t] = (k < E) ? l[order[k - 1]] - l[order[k]] : std::numeric_limits<double>::infinity();
    }
  });
}

// ---------------------------------------------------------------------------
// Token -> expert grouping ([R-zh] sec. 4: only a subset of experts runs per
// token).  Pairs (t, slot) are listed per expert, experts ascending, tokens
// ascending within an expert (a token meets an expert at most once, so the
// order is unique):
//   counts[e], offsets[e] = sum_{e'<e} counts[e'] (offsets[E] = T*k),
//   perm[p] = t*k + slot of the p-th pair in that order, inv[t*k + slot] = p.
// Returns 0, or 1 if an index is out of range or a token repeats an expert.
// ---------------------------------------------------------------------------
int32_t oracle_group(int32_t T, int32_t k, int32_t E, const int32_t* idx, int32_t* counts, int32_t* offsets,
                     int32_t* perm, int32_t* inv) {
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t q = 0; q < (int64_t)T * k; ++q) {
    const int32_t e = idx[q];
    if (e < 0 || e >= E) return 1;
    counts[e]++;
  }
  for (int32_t t = 0; t < T; ++t)
    for (int32_t a = 0; a < k; ++a)
      for (int32_t b = a + 1; b < k; ++b)
        if (idx[(int64_t)t * k + a] == idx[(int64_t)t * k + b]) return 1;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int64_t p = 0;
  for (int32_t e = 0; e < E; ++e)
    for (int32_t t = 0; t < T; ++t)
      for (int32_t s = 0; s < k; ++s)
        if (idx[(int64_t)t * k + s] == e) {
          perm[p] = t * k + s;
          inv[(int64_t)t * k + s] = (int32_t)p;
          ++p;
        }
  return 0;
}

// ---------------------------------------------------------------------------
// One expert's SwiGLU MLP on one bf16-rounded input row ([R-zh] sec. 3:
// three linears, Swish = x*sigmoid(x); [ATLAS] hidden_act silu,
// swiglu_limit 7).  w1: decoded [2I][d] (gate rows then up rows), w2: decoded
// [d][I].  h is rounded to bf16; o is returned unrounded.
// ---------------------------------------------------------------------------
static void expert_mlp(int32_t d, int32_t I, const double* w1, const double* w2, const double* xe, double limit,
                       int32_t act_format, double* h, double* o) {
  for (int32_t n = 0; n < I; ++n) {
    double g = 0.0, u = 0.0;
    for (int32_t i = 0; i < d; ++i) g += w1[(int64_t)n * d + i] * xe[i];
    for (int32_t i = 0; i < d; ++i) u += w1[(int64_t)(I + n) * d + i] * xe[i];
    const double gc = std::min(g, limit);
    const double uc = std::min(std::max(u, -limit), limit);
    h[n] = round_to_bf16(silu(gc) * uc);
  }
  if (act_format)   // low-precision activations: the down projection reads h in 32-blocks along I
    for (int32_t b = 0; b < I / 32; ++b) quantize_activation_block(h + 32 * b, act_format);
  for (int32_t m = 0; m < d; ++m) {
    double acc = 0.0;
    for (int32_t n = 0; n < I; ++n) acc += w2[(int64_t)m * I + n] * h[n];
    o[m] = acc;
  }
}

// ---------------------------------------------------------------------------
// The whole layer for a subset of tokens (rows are independent):
//   xn = RMSNorm(x); (idx, w) = route(xn); xe = bf16(xn)
//   y  = bf16(x + sum_j w_j * Expert_{idx_j}(xe)),  j = 0..k-1 in slot order
// Weights: MXFP4 in the oracle layout, all E experts:
//   w1 codes [E][2I][d/2], scales [E][2I][d/32]; w2 codes [E][d][I/2], scales [E][d][I/32].
// tok: the token ids to compute (n_tok of them; NULL = all T in order).
// Outputs per computed token (row r = position in tok): y_bf16 [n][d];
// optional: y_f64 [n][d] (before the final rounding), idx [n][k], w [n][k],
// h_bf16 [n][k][I] (the rounded SwiGLU outputs as the down projection reads them, slot
// order).  act_format 0: bf16 activations; 1: MXFP8, 2: MXFP4 activations (xe and h quantized in
// 32-blocks, see the header).
// Returns 0, or nonzero on bad arguments / NaN scale bytes.
// ---------------------------------------------------------------------------
int32_t oracle_moe_forward(int32_t T, int32_t d, int32_t I, int32_t E, int32_t k, double eps, double limit,
                           const uint16_t* x, const float* gamma, const float* router_w, const float* router_b,
                           const uint8_t* w1_codes, const uint8_t* w1_scales, const uint8_t* w2_codes,
                           const uint8_t* w2_scales, const int32_t* tok, int32_t n_tok, uint16_t* y_bf16,
                           double* y_f64, int32_t* idx_out, double* w_out, uint16_t* h_bf16, int32_t nthreads,
                           int32_t act_format) {
  if (d % 32 || I % 32 || k < 1 || k > E || act_format < 0 || act_format > 2) return 2;
  if (!tok) n_tok = T;
  std::vector<int32_t> ids(n_tok);
  for (int32_t r = 0; r < n_tok; ++r) ids[r] = tok ? tok[r] : r;
  for (int32_t r = 0; r < n_tok; ++r)
    if (ids[r] < 0 || ids[r] >= T) return 2;

  // Route the selected tokens.
  std::vector<uint16_t> xs((size_t)n_tok * d);
  for (int32_t r = 0; r < n_tok; ++r) std::memcpy(&xs[(size_t)r * d], x + (int64_t)ids[r] * d, 2 * (size_t)d);
  std::vector<int32_t> idx((size_t)n_tok * k);
  std::vector<double> w((size_t)n_tok * k);
  oracle_route(n_tok, d, E, k, xs.data(), gamma, eps, router_w, router_b, idx.data(), w.data(), nullptr, nullptr,
               nthreads);

  // Expert inputs xe = bf16(RMSNorm(x)).
  std::vector<double> xe((size_t)n_tok * d);
  oracle_rmsnorm(n_tok, d, xs.data(), gamma, eps, xe.data());
  for (auto& v : xe) v = round_to_bf16(v);
  if (act_format)
    for (int64_t b = 0; b < (int64_t)n_tok * (d / 32); ++b) quantize_activation_block(&xe[(size_t)b * 32], act_format);

  // Per (token, slot) expert outputs, computed expert by expert so that each
  // expert's weights are decoded once.
  std::vector<double> o((size_t)n_tok * k * d);
  std::vector<double> w1((size_t)2 * I * d), w2((size_t)d * I);
  int32_t status = 0;
  for (int32_t e = 0; e < E; ++e) {
    std::vector<int64_t> jobs;  // r * k + slot
    for (int32_t r = 0; r < n_tok; ++r)
      for (int32_t s = 0; s < k; ++s)
        if (idx[(size_t)r * k + s] == e) jobs.push_back((int64_t)r * k + s);
    if (jobs.empty()) continue;
    status |= oracle_dequantize(w1_codes + (int64_t)e * 2 * I * (d / 2), w1_scales + (int64_t)e * 2 * I * (d / 32),
                                2 * I, d, w1.data());
    status |= oracle_dequantize(w2_codes + (int64_t)e * d * (I / 2), w2_scales + (int64_t)e * d * (I / 32), d, I,
                                w2.data());
    parallel_chunks((int64_t)jobs.size(), nthreads, [&](int64_t j0, int64_t j1) {
      std::vector<double> h(I);
      for (int64_t j = j0; j < j1; ++j) {
        const int64_t q = jobs[j];
        const int64_t r = q / k;
        expert_mlp(d, I, w1.data(), w2.data(), &xe[(size_t)r * d], limit, act_format, h.data(),
                   &o[(size_t)q * d]);
        if (h_bf16)
          for (int32_t n = 0; n < I; ++n) h_bf16[(size_t)q * I + n] = bf16_bits_of(h[n]);
      }
    });
  }

  // Weighted combine + residual ([ARCH] 混合专家模型: weighted sum of the
  // chosen experts; Transformer 块: the block maps [N x d] to [N x d]).
  for (int32_t r = 0; r < n_tok; ++r)
    for (int32_t i = 0; i < d; ++i) {
      double acc = bf16_bits_to_double(xs[(size_t)r * d + i]);
      for (int32_t s = 0; s < k; ++s) acc += w[(size_t)r * k + s] * o[((size_t)r * k + s) * d + i];
      if (y_f64) y_f64[(size_t)r * d + i] = acc;
      y_bf16[(size_t)r * d + i] = bf16_bits_of(round_to_bf16(acc));
    }
  if (idx_out) std::memcpy(idx_out, idx.data(), sizeof(int32_t) * idx.size());
  if (w_out) std::memcpy(w_out, w.data(), sizeof(double) * w.size());
  return status ? 3 : 0;
}

}  // extern "C"
