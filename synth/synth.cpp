// Seeded synthetic input generator shared by the tests, the benchmark and the
// oracle drivers.  It holds none of the MoE layer's arithmetic: it only draws
// numbers.
//
// Every value is a pure function of (seed, stream, sub, index), so any slice of
// any tensor can be regenerated on its own (one token row, one expert matrix)
// and in parallel.
//
// Random bits: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014).  The generator state after i
// steps is  key + (i+1) * GAMMA  and the output is the SplitMix64 mixing
// function of that state, so the i-th draw needs no sequential walk.
// Normals: Box-Muller on consecutive pairs of uniforms.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;  // SplitMix64 increment

inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Key of one substream.  Each argument goes through the mixer so that nearby
// (seed, stream, sub) triples give unrelated keys.
inline uint64_t stream_key(uint64_t seed, uint64_t stream, uint64_t sub) {
  uint64_t k = mix64(seed + kGamma);
  k = mix64(k ^ (stream * 0xD1B54A32D192ED03ull + kGamma));
  k = mix64(k ^ (sub * 0xA0761D6478BD642Full + 0x94D049BB133111EBull));
  return k;
}

inline uint64_t draw_u64(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * kGamma); }

// Uniform in the open interval (0, 1): 53 random bits, offset by half a step.
inline double draw_unit(uint64_t key, uint64_t i) {
  return ((double)(draw_u64(key, i) >> 11) + 0.5) * 0x1.0p-53;
}

// Standard normal number i of the substream: element 2j and 2j+1 share the
// uniform pair (2j, 2j+1).
inline double draw_normal(uint64_t key, uint64_t i) {
  const uint64_t j = i >> 1;
  const double u1 = draw_unit(key, 2 * j);
  const double u2 = draw_unit(key, 2 * j + 1);
  const double r = std::sqrt(-2.0 * std::log(u1));
  const double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * std::sin(a) : r * std::cos(a);
}

inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16);  // inf / nan
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

template <class F>
void parallel_for(int64_t count, int nthreads, F&& body) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  const int64_t min_chunk = 1 << 16;
  int64_t nt = std::min<int64_t>(nthreads, (count + min_chunk - 1) / min_chunk);
  if (nt <= 1) {
    body(0, count);
    return;
  }
  std::vector<std::thread> ts;
  const int64_t chunk = (count + nt - 1) / nt;
  for (int64_t t = 0; t < nt; ++t) {
    const int64_t b = t * chunk, e = std::min(count, b + chunk);
    if (b >= e) break;
    ts.emplace_back([&body, b, e] { body(b, e); });
  }
  for (auto& t : ts) t.join();
}

}  // namespace

extern "C" {

// out[i] = mean + std * N_i for i in [0, count), where N_i is draw (offset + i)
// of substream (seed, stream, sub); rounded once from double to float.
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t sub, uint64_t offset, int64_t count,
                      double mean, double std_, float* out, int nthreads) {
  const uint64_t key = stream_key(seed, stream, sub);
  parallel_for(count, nthreads, [&](int64_t b, int64_t e) {
    for (int64_t i = b; i < e; ++i) out[i] = (float)(mean + std_ * draw_normal(key, offset + (uint64_t)i));
  });
}

// As synth_normal_f32, then rounded to bfloat16 (round to nearest even).
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t sub, uint64_t offset, int64_t count,
                       double mean, double std_, uint16_t* out, int nthreads) {
  const uint64_t key = stream_key(seed, stream, sub);
  parallel_for(count, nthreads, [&](int64_t b, int64_t e) {
    for (int64_t i = b; i < e; ++i)
      out[i] = f32_to_bf16_rne((float)(mean + std_ * draw_normal(key, offset + (uint64_t)i)));
  });
}

// Uniform doubles in (0, 1).
void synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t sub, uint64_t offset, int64_t count,
                       double* out) {
  const uint64_t key = stream_key(seed, stream, sub);
  for (int64_t i = 0; i < count; ++i) out[i] = draw_unit(key, offset + (uint64_t)i);
}

// A uniformly random permutation of 0..n-1 (Fisher-Yates, draws from the
// substream in order; the modulo bias of 64-bit draws is below 2^-40 for n < 2^24).
void synth_permutation(uint64_t seed, uint64_t stream, uint64_t sub, int32_t n, int32_t* out) {
  const uint64_t key = stream_key(seed, stream, sub);
  for (int32_t i = 0; i < n; ++i) out[i] = i;
  for (int32_t i = n - 1; i > 0; --i) {
    const uint64_t r = draw_u64(key, (uint64_t)(n - 1 - i));
    const int32_t j = (int32_t)(r % (uint64_t)(i + 1));
    std::swap(out[i], out[j]);
  }
}

// Raw 64-bit draws (for tests of the generator itself).
void synth_u64(uint64_t seed, uint64_t stream, uint64_t sub, uint64_t offset, int64_t count, uint64_t* out) {
  const uint64_t key = stream_key(seed, stream, sub);
  for (int64_t i = 0; i < count; ++i) out[i] = draw_u64(key, offset + (uint64_t)i);
}

// The SplitMix64 sequence from a plain 64-bit seed, as published: state += GAMMA,
// output = mix(state).  Used by the tests to check mix64 against known values.
void synth_splitmix64_sequence(uint64_t seed, int64_t count, uint64_t* out) {
  uint64_t s = seed;
  for (int64_t i = 0; i < count; ++i) {
    s += kGamma;
    out[i] = mix64(s);
  }
}

}  // extern "C"
