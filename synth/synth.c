/* Counter-based SplitMix64 generators for the synthetic inputs (host only, OpenMP).
 *
 * The same definitions as synth/__init__.py: value i of the (seed, rank, stream)
 * sequence is mix(key + (i + 1) * GOLDEN), mix = the SplitMix64 finaliser
 * (Steele, Lea and Flood, OOPSLA 2014). Compiled without fast-math so that the
 * fp64 Box-Muller transform rounds the way the C library does.
 */
#include <math.h>
#include <stdint.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t synth_stream_key(uint64_t seed, int64_t rank, int64_t stream) {
  uint64_t s = mix(seed);
  return mix(s + (uint64_t)(rank + 1) * GOLDEN + (uint64_t)(stream & 0xFFFFFFFF));
}

void synth_raw_u64(uint64_t key, uint64_t start, int64_t count, uint64_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = mix(key + (start + (uint64_t)i + 1) * GOLDEN);
}

void synth_uniform_f32(uint64_t key, uint64_t start, int64_t count, double lo, double hi, float* out) {
  const int unit = (lo == -1.0 && hi == 1.0);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    uint64_t z = mix(key + (start + (uint64_t)i + 1) * GOLDEN);
    float f = (float)(z >> 40) * 0x1p-24f;
    out[i] = unit ? f * 2.0f - 1.0f : (float)(lo + (hi - lo) * (double)f);
  }
}

void synth_normal_f32(uint64_t key, uint64_t start, int64_t count, double std, float* out) {
  const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    uint64_t z = mix(key + (start + (uint64_t)i + 1) * GOLDEN);
    double u1 = ((double)(z >> 32) + 1.0) * 0x1p-32;
    double u2 = (double)(z & 0xFFFFFFFFULL) * 0x1p-32;
    double g = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
    out[i] = (float)(g * std);
  }
}

void synth_int32(uint64_t key, uint64_t start, int64_t count, int64_t lo, int64_t hi, int32_t* out) {
  const uint64_t span = (uint64_t)(hi - lo + 1);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    uint64_t z = mix(key + (start + (uint64_t)i + 1) * GOLDEN);
    out[i] = (int32_t)((int64_t)(z % span) + lo);
  }
}

void synth_to_bf16(const float* x, int64_t count, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    union { float f; uint32_t u; } v;
    v.f = x[i];
    uint32_t b = v.u;
    out[i] = (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
  }
}
