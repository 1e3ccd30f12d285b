/*
 * synth.c -- seeded synthetic inputs for the quantised MoE expert forward.
 *
 * This module is shared input generation only: it holds none of the
 * method's arithmetic (no dequantisation, no dot products, no routing).
 * Both the CUDA path's tests/benchmarks and the CPU oracle draw their
 * inputs from here, so the two sides see bit-identical tensors.
 *
 * Generator: a counter-based stream built on the SplitMix64 output
 * function (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014):
 *     mix64(z): z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *               z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31.
 * A stream is identified by a 64-bit key derived from (seed, kind, layer,
 * slot); element i of the stream is mix64(key + (i + 1) * GOLDEN), with
 * GOLDEN = 0x9E3779B97F4A7C15.  Any tensor of any layer/expert can thus be
 * regenerated on demand, in any order, on any number of threads.
 *
 * Value recipes (all in the logical, unpacked layout):
 *   codes      element n of a [rows][cols] matrix of b-bit codes is field
 *              (n mod 64/b) of word n / (64/b): uniform in 0 .. 2^b - 1.
 *   uniform    u = (word >> 11) * 2^-53 in [0, 1).
 *   normal     Box-Muller on words 2n, 2n+1: sqrt(-2 ln u1) cos(2 pi u2),
 *              u1 = ((w >> 11) + 1) * 2^-53 in (0, 1].
 *   bf16       round-to-nearest-even of the float32 value.
 *   scale      bf16(lo + (hi - lo) u).
 *   bias       int4: bf16(-8 s + N(0, sigma)), int2: bf16(-1.5 s), with s the
 *              stored (bf16) scale.
 *   zipf/gumbel  per step: a seeded permutation of the experts maps ranks
 *              to ids; token t's logit for the expert at rank r is
 *              log(1/r) - log(-log u) (Gumbel-top-k sampling, Kool et al.
 *              2019), so the top-k of those logits draws k distinct experts
 *              with probability proportional to 1/r.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

uint64_t synth_key(uint64_t seed, uint32_t kind, uint32_t layer, uint32_t slot) {
  uint64_t k = mix64(seed + SYNTH_GOLDEN);
  k = mix64(k ^ (uint64_t)kind);
  k = mix64(k ^ ((uint64_t)layer << 20));
  k = mix64(k ^ ((uint64_t)slot << 40));
  return k;
}

static inline uint64_t word_at(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * SYNTH_GOLDEN);
}

static inline double uniform01(uint64_t w) { return (double)(w >> 11) * 0x1.0p-53; }

static inline double normal_at(uint64_t key, uint64_t n) {
  double u1 = ((double)(word_at(key, 2 * n) >> 11) + 1.0) * 0x1.0p-53;
  double u2 = uniform01(word_at(key, 2 * n + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Raw words, for tests of the stream itself. */
void synth_words(uint64_t key, uint64_t first, uint64_t n, uint64_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = word_at(key, first + i);
}

/* Uniform b-bit codes for elements [first, first + n) of a stream. */
void synth_codes(uint64_t key, int bits, uint64_t first, uint64_t n, uint8_t* out) {
  const uint64_t per_word = 64u / (uint64_t)bits;
  const uint64_t mask = (1ULL << bits) - 1ULL;
  uint64_t i = 0;
  while (i < n) {
    uint64_t e = first + i;
    uint64_t w = word_at(key, e / per_word);
    uint64_t f = e % per_word;
    for (; f < per_word && i < n; ++f, ++i) out[i] = (uint8_t)((w >> (bits * f)) & mask);
  }
}

/* Scale and bias (bf16 bits) for n groups starting at group index first.
 * bits == 4: bias = bf16(-8 s + N(0, bias_sigma)); bits == 2: bf16(-1.5 s). */
void synth_scale_bias(uint64_t key_scale, uint64_t key_bias, int bits, double lo, double hi,
                      double bias_sigma, uint64_t first, uint64_t n, uint16_t* scale,
                      uint16_t* bias) {
  for (uint64_t i = 0; i < n; ++i) {
    uint64_t g = first + i;
    double u = uniform01(word_at(key_scale, g));
    uint16_t sb = f32_to_bf16_rne((float)(lo + (hi - lo) * u));
    double s = (double)bf16_to_f32(sb);
    double b;
    if (bits == 4)
      b = -8.0 * s + bias_sigma * normal_at(key_bias, g);
    else
      b = -1.5 * s;
    scale[i] = sb;
    bias[i] = f32_to_bf16_rne((float)b);
  }
}

/* out[i] = float(mean + std * N(0,1)) for elements [first, first + n). */
void synth_normal_f32(uint64_t key, double mean, double std, uint64_t first, uint64_t n,
                      float* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, first + i));
}

/* Zipf(1) popularity over n_experts with Gumbel noise, as router logits for
 * n_tokens tokens of one step: logits[t * n_experts + id]. perm_key fixes the
 * rank -> id permutation; noise_key the per-token Gumbel draws. */
void synth_zipf_gumbel_logits(uint64_t perm_key, uint64_t noise_key, int n_tokens,
                              int n_experts, float* logits, int32_t* rank_to_id) {
  for (int i = 0; i < n_experts; ++i) rank_to_id[i] = i;
  for (int i = n_experts - 1; i > 0; --i) { /* Fisher-Yates */
    uint64_t j = word_at(perm_key, (uint64_t)i) % (uint64_t)(i + 1);
    int32_t t = rank_to_id[i];
    rank_to_id[i] = rank_to_id[j];
    rank_to_id[j] = t;
  }
  for (int t = 0; t < n_tokens; ++t) {
    for (int r = 0; r < n_experts; ++r) {
      uint64_t idx = (uint64_t)t * (uint64_t)n_experts + (uint64_t)r;
      double u1 = ((double)(word_at(noise_key, idx) >> 11) + 1.0) * 0x1.0p-53; /* (0,1] */
      if (u1 >= 1.0) u1 = 1.0 - 0x1.0p-53;
      double gumbel = -log(-log(u1));
      logits[(size_t)t * n_experts + rank_to_id[r]] = (float)(-log((double)(r + 1)) + gumbel);
    }
  }
}

/* bf16 helpers exposed for the Python side (rounding of inputs only). */
void synth_f32_to_bf16(const float* in, uint64_t n, uint16_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}
