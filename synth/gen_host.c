/*
 * Seeded synthetic inputs, host side.
 *
 * This file is an input generator and holds none of the MoE layer's
 * arithmetic.  A twin written separately for the GPU (gen_device.cu) draws
 * the same numbers from the same definition, so a large weight tensor can be
 * generated on the device and any slice of it regenerated on the host.
 *
 * Definition (both sides implement exactly this, from the published
 * algorithms named here):
 *
 *   mix64(z)   SplitMix64 output function (Steele, Lea and Flood, "Fast
 *              splittable pseudorandom number generators", OOPSLA 2014; the
 *              constants are those of Vigna's public-domain splitmix64.c):
 *                z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *                z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *                return z ^ (z >> 31)
 *   GAMMA      0x9E3779B97F4A7C15 (the SplitMix64 increment)
 *   key(seed, stream) = mix64(seed * GAMMA ^ mix64(stream + GAMMA))
 *   draw(key, i)      = mix64(key + (i + 1) * GAMMA)      (i-th output of a
 *                       SplitMix64 sequence whose state starts at key)
 *
 *   normal(key, i): the classic "sum of twelve uniforms minus six"
 *   (Irwin-Hall, n = 12) approximation of N(0, 1).  The twelve uniforms are
 *   the four 16-bit fields of each of draw(key, 3i), draw(key, 3i+1),
 *   draw(key, 3i+2); with S their integer sum,
 *                z = (float)(S - 393210) * 2^-16        (exact in fp32)
 *   so z has mean 0, variance 1 - 2^-32 and support [-6, 6).
 *
 *   normal_bf16(key, i, sigma) = bf16_rne(z * sigma)   one fp32 multiply
 *                                (round to nearest), then round-to-nearest-even
 *                                of the fp32 bit pattern to bf16.
 *   normal_f32(key, i, sigma)  = z * sigma              in fp32.
 *   uniform_int(key, i, n)     = ((draw(key, i) >> 32) * n) >> 32   in [0, n).
 *
 * All arithmetic is integer except one correctly rounded fp32 multiply, so
 * the host and device twins agree bit for bit.  Compile with
 * -ffp-contract=off (there is nothing to contract, but the flag keeps it so).
 */
#include <stdint.h>
#include <string.h>

#define SYN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t syn_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t syn_key(uint64_t seed, uint64_t stream) {
  return syn_mix64((seed * SYN_GAMMA) ^ syn_mix64(stream + SYN_GAMMA));
}

uint64_t syn_draw(uint64_t key, uint64_t i) {
  return syn_mix64(key + (i + 1) * SYN_GAMMA);
}

static inline float syn_z(uint64_t key, uint64_t i) {
  int32_t s = 0;
  for (int j = 0; j < 3; ++j) {
    uint64_t d = syn_draw(key, 3 * i + (uint64_t)j);
    s += (int32_t)(d & 0xFFFF) + (int32_t)((d >> 16) & 0xFFFF) +
         (int32_t)((d >> 32) & 0xFFFF) + (int32_t)(d >> 48);
  }
  return (float)(s - 393210) * (1.0f / 65536.0f);
}

static inline uint16_t syn_f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* out[j] = normal_bf16(key, start + j, sigma), j < count */
void syn_normal_bf16(uint64_t key, uint64_t start, uint64_t count, float sigma,
                     uint16_t *out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)count; ++j)
    out[j] = syn_f32_to_bf16_rne(syn_z(key, start + (uint64_t)j) * sigma);
}

/* The same bf16 draws, each widened exactly to double (a storage format only:
 * the bf16 value placed in the upper half of an fp32 pattern, then converted). */
void syn_normal_bf16_as_f64(uint64_t key, uint64_t start, uint64_t count, float sigma,
                            double *out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)count; ++j) {
    uint32_t u = (uint32_t)syn_f32_to_bf16_rne(syn_z(key, start + (uint64_t)j) * sigma) << 16;
    float f;
    memcpy(&f, &u, 4);
    out[j] = (double)f;
  }
}

void syn_normal_f32(uint64_t key, uint64_t start, uint64_t count, float sigma,
                    float *out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)count; ++j)
    out[j] = syn_z(key, start + (uint64_t)j) * sigma;
}

void syn_uniform_int(uint64_t key, uint64_t start, uint64_t count, uint32_t n,
                     int32_t *out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)count; ++j)
    out[j] = (int32_t)(((syn_draw(key, start + (uint64_t)j) >> 32) * (uint64_t)n) >> 32);
}

/* The raw SplitMix64 sequence from a seed, for checking mix64 against the
 * published reference outputs: out[j] = mix64(seed + (j + 1) * GAMMA). */
void syn_splitmix64_sequence(uint64_t seed, uint64_t count, uint64_t *out) {
  for (uint64_t j = 0; j < count; ++j) out[j] = syn_mix64(seed + (j + 1) * SYN_GAMMA);
}
