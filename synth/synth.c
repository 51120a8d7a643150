/*
 * Seeded, counter-based input generator for GR-KAN workloads.
 *
 * This file draws random numbers and nothing else: it holds none of the
 * activation's arithmetic. Both the fp64 oracle and the CUDA path read the
 * buffers it writes, so the two sides always see the same inputs.
 *
 * Definition (stated so that any implementation can reproduce it):
 *   mix64(z)          : the SplitMix64 output function
 *                       z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                       z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31
 *   key(seed, stream) = mix64(seed*0x9E3779B97F4A7C15 + stream*0xD1B54A32D192ED03 + 1)
 *   bits(seed, stream, i) = mix64(key + (i+1)*0x9E3779B97F4A7C15)   (mod 2^64)
 *   uniform(i)  = (bits >> 11) * 2^-53                      in [0, 1)
 *   normal(i)   = sqrt(-2 ln(1 - uniform(2i))) * cos(2 pi uniform(2i+1))
 *   student3(i) = normal(4i) / sqrt((normal(4i+1)^2 + normal(4i+2)^2 + normal(4i+3)^2) / 3)
 * Every draw is computed in double, rounded to float32 (round to nearest even),
 * and for bf16 outputs the float32 value is rounded to bf16 (nearest even).
 * Element i of a tensor depends only on (seed, stream, i), so any slice can be
 * regenerated alone and the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define SYN_F32 0
#define SYN_BF16 1

static const double SYN_TWO_PI = 6.283185307179586476925286766559;

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed * 0x9E3779B97F4A7C15ULL + stream * 0xD1B54A32D192ED03ULL + 1ULL);
}

static inline double uniform_at(uint64_t key, uint64_t i) {
  uint64_t z = mix64(key + (i + 1ULL) * 0x9E3779B97F4A7C15ULL);
  return (double)(z >> 11) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  double u1 = uniform_at(key, 2ULL * i);
  double u2 = uniform_at(key, 2ULL * i + 1ULL);
  return sqrt(-2.0 * log(1.0 - u1)) * cos(SYN_TWO_PI * u2);
}

static inline double student3_at(uint64_t key, uint64_t i) {
  double z0 = normal_at(key, 4ULL * i);
  double z1 = normal_at(key, 4ULL * i + 1ULL);
  double z2 = normal_at(key, 4ULL * i + 2ULL);
  double z3 = normal_at(key, 4ULL * i + 3ULL);
  return z0 / sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline void store(void* out, int dtype, int64_t j, double v) {
  float f = (float)v;
  if (dtype == SYN_F32)
    ((float*)out)[j] = f;
  else
    ((uint16_t*)out)[j] = f32_to_bf16_rne(f);
}

/* kind: 0 = normal*scale, 1 = student-t(3) clipped to [-clip, clip] then *scale,
 *       2 = uniform in [lo, hi) (scale=lo, clip=hi).
 * Writes elements [offset, offset+count) of the tensor to out[0..count). */
int synth_fill(uint64_t seed, uint64_t stream, int kind, int64_t offset, int64_t count, double scale,
               double clip, int dtype, void* out, int nthreads) {
  if (count < 0 || offset < 0 || (dtype != SYN_F32 && dtype != SYN_BF16) || kind < 0 || kind > 2)
    return 1;
  uint64_t key = stream_key(seed, stream);
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
  for (int64_t j = 0; j < count; ++j) {
    uint64_t i = (uint64_t)(offset + j);
    double v;
    if (kind == 0) {
      v = scale * normal_at(key, i);
    } else if (kind == 1) {
      double t = student3_at(key, i);
      if (t > clip) t = clip;
      if (t < -clip) t = -clip;
      v = scale * t;
    } else {
      v = scale + (clip - scale) * uniform_at(key, i);
    }
    store(out, dtype, j, v);
  }
  (void)nthreads;
  return 0;
}

/* Gather variant: writes element idx[j] of the tensor to out[j]. */
int synth_fill_at(uint64_t seed, uint64_t stream, int kind, const int64_t* idx, int64_t count,
                  double scale, double clip, int dtype, void* out) {
  if (count < 0 || (dtype != SYN_F32 && dtype != SYN_BF16) || kind < 0 || kind > 2) return 1;
  uint64_t key = stream_key(seed, stream);
  for (int64_t j = 0; j < count; ++j) {
    uint64_t i = (uint64_t)idx[j];
    double v;
    if (kind == 0) {
      v = scale * normal_at(key, i);
    } else if (kind == 1) {
      double t = student3_at(key, i);
      if (t > clip) t = clip;
      if (t < -clip) t = -clip;
      v = scale * t;
    } else {
      v = scale + (clip - scale) * uniform_at(key, i);
    }
    store(out, dtype, j, v);
  }
  return 0;
}

int synth_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
