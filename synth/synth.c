/*
 * Seeded synthetic-input generator shared by the tests, the bench and the
 * oracle checks.  It holds no MoE arithmetic: it only turns (seed, stream,
 * element index) into a normally distributed number and rounds it to the
 * storage type.
 *
 * Definition (so that any other implementation can reproduce it bit for bit):
 *   mix64(z)      = SplitMix64 output function (Steele, Lea, Flood, "Fast
 *                   splittable pseudorandom number generators", OOPSLA 2014):
 *                   z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                   z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31
 *   key(seed,s)   = mix64(seed * 0x9E3779B97F4A7C15 + mix64(s + 0x632BE59BD9B4E019))
 *   word(i)       = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   unif(i)       = ((word(i) >> 11) + 1) * 2^-53            in (0, 1]
 *   pair j        : r = sqrt(-2 ln unif(2j)), a = 2*pi*unif(2j+1)
 *   normal(2j)    = r cos a,  normal(2j+1) = r sin a          (Box-Muller)
 *   value(i)      = mean + std * normal(i), computed in double,
 *                   rounded to float (round-to-nearest-even), and for bf16
 *                   storage rounded once more from float to bf16 (RNE).
 * Counter based: element i depends only on (seed, stream, i), so any slice
 * can be regenerated independently and the work splits across threads.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed * GOLDEN + mix64(stream + 0x632BE59BD9B4E019ULL));
}

static inline double unif(uint64_t key, uint64_t i) {
  uint64_t w = mix64(key + (i + 1) * GOLDEN);
  return (double)((w >> 11) + 1) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  uint64_t j = i >> 1;
  double u1 = unif(key, 2 * j);
  double u2 = unif(key, 2 * j + 1);
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu)) return (uint16_t)((b >> 16) | 0x40);
  uint32_t lsb = (b >> 16) & 1u;
  b += 0x7FFFu + lsb;
  return (uint16_t)(b >> 16);
}

/* n values of mean + std*N(0,1) as float, elements [offset, offset+n) of the stream */
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean, double std,
                      float* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, offset + (uint64_t)i));
}

/* same values, stored as bf16 bit patterns */
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean, double std,
                       uint16_t* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = f32_to_bf16_rne((float)(mean + std * normal_at(key, offset + (uint64_t)i)));
}

/* raw 64-bit words, exposed so that the generator itself can be tested */
void synth_words(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint64_t* out) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = mix64(key + (offset + (uint64_t)i + 1) * GOLDEN);
}

/* float -> bf16 (RNE) for arrays the caller built itself (e.g. closed-form inputs) */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}
