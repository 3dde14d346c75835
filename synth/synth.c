/*
 * Seeded synthetic inputs for the GQA forward: the one module that both the
 * fp64 oracle (through the tests) and the CUDA path (through the tests and the
 * benchmark) draw their inputs from.  It holds none of the attention
 * arithmetic: only a counter-based random number generator, the standard
 * normal transform and the rounding of fp32 values to bf16.
 *
 * Generator.  SplitMix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-style: the
 * i-th output (i = 0, 1, ...) of the stream seeded with `key` is
 * mix(key + (i + 1) * GAMMA), which is exactly what the sequential generator
 * returns on its (i+1)-th call.  Because every output is a pure function of
 * (key, i), any slice of a tensor can be produced on its own, on any thread,
 * and always gives the same bits.
 *
 * Normal deviates.  Box and Muller ("A note on the generation of random
 * normal deviates", Ann. Math. Statist. 1958): one 64-bit output gives two
 * 32-bit uniforms u1 in (0, 1] and u2 in [0, 1); element 2p of a tensor is
 * R cos(theta) and element 2p+1 is R sin(theta), with R = sqrt(-2 ln u1) and
 * theta = 2 pi u2, evaluated in double and rounded to float.
 *
 * bf16.  Round-to-nearest-even of the float's upper 16 bits, done on the bit
 * pattern (the inputs are finite, so no NaN handling is needed).
 *
 * Flat element index e of a tensor is its position in the logical contiguous
 * [B, H, S, D] order; `offset` lets a caller produce elements
 * [offset, offset + count) only.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t synth_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* i-th output of the SplitMix64 stream seeded with key. */
static inline uint64_t synth_at(uint64_t key, uint64_t i) {
  return synth_mix(key + (i + 1ULL) * SYNTH_GAMMA);
}

/* Key of sub-stream `stream` (0 = Q, 1 = K, 2 = V, 3 = mask, ...) of `seed`. */
uint64_t synth_stream_key(uint64_t seed, uint64_t stream) {
  return synth_at(synth_at(seed, 0), stream);
}

uint64_t synth_u64(uint64_t key, uint64_t i) { return synth_at(key, i); }

static inline double synth_normal_at(uint64_t key, uint64_t e) {
  const uint64_t r = synth_at(key, e >> 1);
  const double two32 = 4294967296.0;
  const double u1 = ((double)(r >> 32) + 1.0) / two32;        /* (0, 1] */
  const double u2 = (double)(r & 0xFFFFFFFFULL) / two32;      /* [0, 1) */
  const double rad = sqrt(-2.0 * log(u1));
  const double theta = 6.283185307179586476925286766559 * u2;
  return (e & 1ULL) ? rad * sin(theta) : rad * cos(theta);
}

static inline uint16_t synth_f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof(u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset,
                      int64_t count, float* out) {
  const uint64_t key = synth_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < count; ++t)
    out[t] = (float)synth_normal_at(key, offset + (uint64_t)t);
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset,
                       int64_t count, uint16_t* out) {
  const uint64_t key = synth_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < count; ++t)
    out[t] = synth_f32_to_bf16_rne((float)synth_normal_at(key, offset + (uint64_t)t));
}

/* Round an fp32 array to bf16 (RNE) bit patterns. */
void synth_round_bf16(const float* in, int64_t count, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < count; ++t) out[t] = synth_f32_to_bf16_rne(in[t]);
}

/* Exact widening of bf16 bit patterns to double. */
void synth_bf16_to_f64(const uint16_t* in, int64_t count, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < count; ++t) {
    uint32_t u = (uint32_t)in[t] << 16;
    float f;
    memcpy(&f, &u, sizeof(f));
    out[t] = (double)f;
  }
}

/* n integers uniform on [lo, hi] (modulo reduction of a 64-bit output). */
void synth_uniform_int(uint64_t seed, uint64_t stream, int64_t n, int64_t lo,
                       int64_t hi, int64_t* out) {
  const uint64_t key = synth_stream_key(seed, stream);
  const uint64_t span = (uint64_t)(hi - lo) + 1ULL;
  for (int64_t t = 0; t < n; ++t) out[t] = lo + (int64_t)(synth_at(key, (uint64_t)t) % span);
}

/* Padding mask of a right-padded batch: mask[b, i, j] = (j < len[b]). */
void synth_mask_lengths(const int64_t* len, int64_t B, int64_t Sq, int64_t Sk,
                        uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < B * Sq; ++r) {
    const int64_t b = r / Sq;
    uint8_t* row = out + r * Sk;
    for (int64_t j = 0; j < Sk; ++j) row[j] = (uint8_t)(j < len[b]);
  }
}

/*
 * Bernoulli(p_true) mask [B, Sq, Sk]; one position per row, chosen from the
 * same stream, is forced true so that no row is fully masked.
 */
void synth_mask_random(uint64_t seed, uint64_t stream, int64_t B, int64_t Sq,
                       int64_t Sk, double p_true, uint8_t* out) {
  const uint64_t key = synth_stream_key(seed, stream);
  const uint64_t thresh = (uint64_t)(p_true * 18446744073709551615.0);
  const int64_t rows = B * Sq;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    uint8_t* row = out + r * Sk;
    for (int64_t j = 0; j < Sk; ++j)
      row[j] = (uint8_t)(synth_at(key, (uint64_t)(r * Sk + j)) < thresh);
    const uint64_t pick = synth_at(key, (uint64_t)(rows * Sk + r)) % (uint64_t)Sk;
    row[pick] = 1;
  }
}
