/*
 * Seeded synthetic input generator shared by the tests, the benchmark and the
 * oracle harness.  It holds none of the MoE layer's arithmetic: it only turns
 * (seed, tensor id, element index) into numbers with a stated distribution.
 *
 * Generator (counter based, so any element can be produced independently and
 * the fill parallelises without changing a single bit):
 *
 *   key(seed, id)  = mix(mix(seed + G) ^ (id * G2))
 *   raw(key, i)    = mix(key + (i + 1) * G)          -- the i-th output of a
 *                                                      SplitMix64 stream whose
 *                                                      state starts at key
 *   mix(z)         = SplitMix64 finaliser (Steele, Lea & Flood, "Fast
 *                    splittable pseudorandom number generators", OOPSLA 2014):
 *                    z ^= z >> 30; z *= 0xbf58476d1ce4e5b9;
 *                    z ^= z >> 27; z *= 0x94d049bb133111eb; z ^= z >> 31
 *   G  = 0x9e3779b97f4a7c15 (golden-ratio increment), G2 = 0xd1b54a32d192ed03
 *
 *   uniform(i)     = ((raw(i) >> 11) + 0.5) * 2^-53                in (0, 1)
 *   normal(i)      = Box-Muller (Box & Muller 1958) on the pair p = i / 2:
 *                    r = sqrt(-2 ln uniform(2p)), a = 2 pi uniform(2p + 1),
 *                    element 2p -> r cos a, element 2p + 1 -> r sin a
 *   int(i; lo, hi) = lo + ((raw(i) >> 32) * (hi - lo + 1)) >> 32   (multiply-shift)
 *
 * Values are computed in double, then rounded once to the stored type:
 * float32 by C's conversion (round to nearest even), bfloat16 by
 * round-to-nearest-even on the float32 bits.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define IG_G 0x9e3779b97f4a7c15ULL
#define IG_G2 0xd1b54a32d192ed03ULL

static inline uint64_t ig_mix(uint64_t z) {
  z ^= z >> 30;
  z *= 0xbf58476d1ce4e5b9ULL;
  z ^= z >> 27;
  z *= 0x94d049bb133111ebULL;
  z ^= z >> 31;
  return z;
}

uint64_t ig_key(uint64_t seed, uint64_t tensor_id) {
  return ig_mix(ig_mix(seed + IG_G) ^ (tensor_id * IG_G2));
}

uint64_t ig_raw(uint64_t key, uint64_t i) { return ig_mix(key + (i + 1) * IG_G); }

static inline double ig_uniform01(uint64_t key, uint64_t i) {
  return ((double)(ig_raw(key, i) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double ig_normal(uint64_t key, uint64_t i) {
  const uint64_t p = i >> 1;
  const double u1 = ig_uniform01(key, 2 * p);
  const double u2 = ig_uniform01(key, 2 * p + 1);
  const double r = sqrt(-2.0 * log(u1));
  const double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t ig_f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Fill out[0..n) with std * N(0,1) as float32. */
void ig_fill_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id, double std) {
  const uint64_t key = ig_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(std * ig_normal(key, (uint64_t)i));
}

/* Fill out[0..n) with std * N(0,1) rounded to bfloat16 (raw bits). */
void ig_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t tensor_id, double std) {
  const uint64_t key = ig_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = ig_f32_to_bf16_rne((float)(std * ig_normal(key, (uint64_t)i)));
}

/* Fill out[0..n) with U(lo, hi) as float32. */
void ig_fill_uniform_f32(float* out, int64_t n, uint64_t seed, uint64_t tensor_id, double lo,
                         double hi) {
  const uint64_t key = ig_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = (float)(lo + (hi - lo) * ig_uniform01(key, (uint64_t)i));
}

/* Fill out[0..n) with integers uniform on [lo, hi] (inclusive) as int8. */
void ig_fill_int8(int8_t* out, int64_t n, uint64_t seed, uint64_t tensor_id, int lo, int hi) {
  const uint64_t key = ig_key(seed, tensor_id);
  const uint64_t span = (uint64_t)(hi - lo + 1);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = (int8_t)(lo + (int)(((ig_raw(key, (uint64_t)i) >> 32) * span) >> 32));
}

/* Threads the fills above may use (OpenMP), for reporting. */
int ig_max_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
