/*
 * Seeded synthetic inputs for the MoE layer: the one module that both the
 * CPU oracle and the CUDA path are fed from.  It holds none of the layer's
 * arithmetic: it only turns (seed, stream, element index) into numbers.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), used counter-style: element i of stream
 * `sid` under seed `seed` is mix(key + (i + 1) * GAMMA) with
 * key = mix(seed ^ mix(sid + GAMMA)).  Being a pure function of the index,
 * any slice can be regenerated and the work splits across threads without
 * changing a single value.
 *   uniform  u = (x >> 11) * 2^-53                in [0, 1)
 *   normal   Box-Muller on the pair (2m, 2m+1):  r = sqrt(-2 ln(1 - u0)),
 *            z0 = r cos(2 pi u1), z1 = r sin(2 pi u1)
 *   bf16     float value rounded to nearest-even on its upper 16 bits.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t sid) {
  return mix64(seed ^ mix64(sid + GAMMA));
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * GAMMA);
}

static inline double unif(uint64_t key, uint64_t i) {
  return (double)(draw(key, i) >> 11) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  uint64_t m = i >> 1;
  double u0 = unif(key, 2 * m), u1 = unif(key, 2 * m + 1);
  double r = sqrt(-2.0 * log(1.0 - u0));
  double a = 6.283185307179586476925286766559 * u1;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16);  /* inf/nan */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t synth_raw(uint64_t seed, uint64_t sid, uint64_t i) { return draw(stream_key(seed, sid), i); }

void synth_normal_bf16(uint64_t seed, uint64_t sid, int64_t n, double mean, double std,
                       uint16_t *out) {
  uint64_t key = stream_key(seed, sid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = f32_to_bf16_rne((float)(mean + std * normal_at(key, (uint64_t)i)));
}

void synth_normal_f32(uint64_t seed, uint64_t sid, int64_t n, double mean, double std, float *out) {
  uint64_t key = stream_key(seed, sid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, (uint64_t)i));
}

void synth_uniform_f32(uint64_t seed, uint64_t sid, int64_t n, double lo, double hi, float *out) {
  uint64_t key = stream_key(seed, sid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(lo + (hi - lo) * unif(key, (uint64_t)i));
}

/* Uniform integers in [0, m): (x >> 11) * m / 2^53, floor. */
void synth_uniform_int(uint64_t seed, uint64_t sid, int64_t n, int64_t m, int64_t *out) {
  uint64_t key = stream_key(seed, sid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (int64_t)(unif(key, (uint64_t)i) * (double)m);
}
