/*
 * Seeded synthetic input streams for the DSA hot path (indexer, top-k,
 * sparse MLA, indexer KL).  This file holds random-number generation only:
 * no step of the method's arithmetic lives here.  Both the CPU oracle's
 * tests and the GPU path's tests/bench draw their inputs from these streams.
 *
 * Generator (stated so that any side can re-implement it):
 *   mix(z)     : z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *                z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *                return z ^ (z >> 31)                  (SplitMix64 finaliser)
 *   key        = mix(seed ^ (tensor_id * 0xD1B54A32D192ED03))
 *   word(i)    = mix(key + (i + 1) * 0x9E3779B97F4A7C15)  (counter-based SplitMix64)
 *   int in [lo,hi] : lo + ((word(i) >> 32) * (hi - lo + 1)) >> 32   (Lemire)
 *   normal pair j  : u1 = ((word(2j) >> 11) + 1) * 2^-53,  u2 = (word(2j+1) >> 11) * 2^-53
 *                    r = sqrt(-2 ln u1); z(2j) = r cos(2 pi u2); z(2j+1) = r sin(2 pi u2)
 *                    (fp64), then rounded to fp32 (RNE), then to bf16 (RNE).
 */
#include <stdint.h>
#include <math.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
  return mix64(seed ^ (tensor_id * 0xD1B54A32D192ED03ULL));
}

static inline uint64_t word_at(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * 0x9E3779B97F4A7C15ULL);
}

/* fp32 -> bf16 with round-to-nearest-even (inputs are finite). */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Elements [offset, offset + n) of each stream; offset of normal streams must be even. */
void dsa_gen_words(uint64_t seed, uint64_t tensor_id, int64_t offset, int64_t n, uint64_t* out) {
  const uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = word_at(key, (uint64_t)(offset + i));
}

void dsa_gen_uniform_int(uint64_t seed, uint64_t tensor_id, int64_t offset, int64_t n, int32_t lo,
                         int32_t hi, int32_t* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  const uint64_t range = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint64_t x = word_at(key, (uint64_t)(offset + i)) >> 32;
    out[i] = lo + (int32_t)((x * range) >> 32);
  }
}

static void normal_pair(uint64_t key, int64_t j, double* z0, double* z1) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  double u1 = (double)((word_at(key, (uint64_t)(2 * j)) >> 11) + 1) * two_m53;
  double u2 = (double)(word_at(key, (uint64_t)(2 * j + 1)) >> 11) * two_m53;
  double r = sqrt(-2.0 * log(u1));
  const double two_pi = 6.283185307179586476925286766559;
  *z0 = r * cos(two_pi * u2);
  *z1 = r * sin(two_pi * u2);
}

void dsa_gen_normal_f64(uint64_t seed, uint64_t tensor_id, int64_t offset, int64_t n, double* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  const int64_t pairs = (n + 1) / 2, j0 = offset / 2;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < pairs; ++j) {
    double a, b;
    normal_pair(key, j0 + j, &a, &b);
    out[2 * j] = a;
    if (2 * j + 1 < n) out[2 * j + 1] = b;
  }
}

void dsa_gen_normal_bf16(uint64_t seed, uint64_t tensor_id, int64_t offset, int64_t n,
                         uint16_t* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  const int64_t pairs = (n + 1) / 2, j0 = offset / 2;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < pairs; ++j) {
    double a, b;
    normal_pair(key, j0 + j, &a, &b);
    out[2 * j] = f32_to_bf16_rne((float)a);
    if (2 * j + 1 < n) out[2 * j + 1] = f32_to_bf16_rne((float)b);
  }
}

/* Integers uniform in [-3, 3] (the int stream with lo=-3, hi=3) stored as OCP e4m3fn bytes:
 * -3 0xC4, -2 0xC0, -1 0xB8, 0 0x00, 1 0x38, 2 0x40, 3 0x44 (exact encodings). */
void dsa_gen_e4m3_small_int(uint64_t seed, uint64_t tensor_id, int64_t offset, int64_t n,
                            uint8_t* out) {
  static const uint8_t enc[7] = {0xC4, 0xC0, 0xB8, 0x00, 0x38, 0x40, 0x44};
  const uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint64_t x = word_at(key, (uint64_t)(offset + i)) >> 32;
    out[i] = enc[(x * 7u) >> 32];
  }
}
