/*
 * Seeded, counter-based synthetic input generator.
 *
 * This file produces the workload inputs (activations, weights, router logits)
 * that both the CUDA path and the CPU oracle consume.  It holds none of the
 * NVFP4 / residual-compensation arithmetic: only random numbers and their
 * conversion to bf16 storage.
 *
 * Generator definition (so that any implementation can reproduce it):
 *   mix64(z)   : the SplitMix64 output finaliser (Steele, Lea & Flood, OOPSLA 2014;
 *                constants as published by S. Vigna):
 *                z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
 *                z *= 0x94D049BB133111EB; z ^= z>>31
 *   key(seed, stream) = mix64(seed ^ mix64(stream + 0x632BE59BD9B4E019))
 *   bits(key, i)      = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   uniform(key, i)   = ((bits >> 11) + 0.5) * 2^-53           in (0, 1)
 *   normal(key, i)    : Box-Muller on the pair p = i >> 1,
 *                       u1 = uniform(key, 2p), u2 = uniform(key, 2p + 1),
 *                       rad = sqrt(-2 ln u1), th = 2 pi u2,
 *                       even i -> rad cos th, odd i -> rad sin th   (double)
 *   bf16 storage      : value computed in double, rounded to float (RN), then to
 *                       bf16 with round-to-nearest-even on the float bits.
 * Every element depends only on (seed, stream, index): results do not depend
 * on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return mix64(seed ^ mix64(stream + 0x632BE59BD9B4E019ULL));
}

static inline double uniform01(uint64_t key, uint64_t i) {
  uint64_t b = mix64(key + (i + 1) * 0x9E3779B97F4A7C15ULL);
  return ((double)(b >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  uint64_t p = i >> 1;
  double u1 = uniform01(key, 2 * p);
  double u2 = uniform01(key, 2 * p + 1);
  double rad = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? rad * sin(th) : rad * cos(th);
}

static inline uint16_t float_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* out[i] = uniform(key(seed, stream), offset + i) */
void synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = uniform01(key, offset + (uint64_t)i);
}

/* out[i] = normal(key(seed, stream), offset + i) */
void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = normal_at(key, offset + (uint64_t)i);
}

/*
 * bf16 matrix [rows x cols], element (r, c) at counter offset + r*cols + c:
 *   out = bf16(float(sigma * colscale[c] * normal))      (colscale may be NULL -> 1)
 */
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t rows, int64_t cols,
                       double sigma, const double* colscale, uint16_t* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      uint64_t idx = offset + (uint64_t)(r * cols + c);
      double v = sigma * normal_at(key, idx);
      if (colscale) v *= colscale[c];
      out[r * cols + c] = float_to_bf16_rne((float)v);
    }
  }
}

int synth_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
