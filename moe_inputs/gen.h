/*
 * Seeded, counter-based synthetic input generator.
 *
 * This header holds no part of the MoE method: it only turns a
 * (seed, tensor id, element index) triple into one number, the same on the
 * host (C, compiled with -ffp-contract=off) and on the GPU (CUDA, with
 * explicitly rounded fp32 operations), so that the CPU oracle and the CUDA
 * path can be fed bit-identical inputs without copying tensors around.
 *
 * Hash: the SplitMix64 output function (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; constants as in Vigna's
 * public-domain splitmix64.c), applied to one state word per element:
 *
 *     state = ((tensor_id << 48) | index) ^ (seed * 0xD1B54A32D192ED03)
 *     h     = splitmix64_next(state)     (i.e. mix(state + golden gamma))
 *
 * With seed = tensor_id = index = 0 the state is 0 and h is SplitMix64's
 * first output for seed 0, 0xE220A8397B1DCDAF (a published test value).
 *
 * Distributions (all arithmetic exact or a single IEEE fp32 rounding):
 *   normal(sigma):  S = sum of the four 16-bit fields of h minus 131070
 *                   (an Irwin-Hall sum, exact int32, mean 0, sd 65536/sqrt 3);
 *                   value = fl32((float)S * c), c = fl32(sigma*sqrt(3)/65536)
 *                   computed by the caller.  Range is +-3.46 sigma.
 *   uniform(a, w):  u = top 24 bits of h; t = u * 2^-24 (exact);
 *                   value = fl32(a + fl32(w * t)), w = fl32(b - a).
 *   constant(a):    value = a.
 * The fp32 value is then stored as fp32, or rounded to bf16 (round to
 * nearest even).
 */
#ifndef MOE_INPUTS_GEN_H
#define MOE_INPUTS_GEN_H

#include <stdint.h>

#ifdef __CUDACC__
#define MOE_GEN_HD __host__ __device__ __forceinline__
#else
#define MOE_GEN_HD static inline
#endif

enum { MOE_GEN_NORMAL = 0, MOE_GEN_UNIFORM = 1, MOE_GEN_CONST = 2 };
enum { MOE_GEN_F32 = 0, MOE_GEN_BF16 = 1 };

MOE_GEN_HD uint64_t moe_gen_hash(uint64_t seed, uint32_t tensor_id, uint64_t index) {
  uint64_t state = (((uint64_t)tensor_id << 48) | (index & 0xFFFFFFFFFFFFull)) ^
                   (seed * 0xD1B54A32D192ED03ull);
  uint64_t z = state + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

MOE_GEN_HD float moe_gen_mul(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}

MOE_GEN_HD float moe_gen_add(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fadd_rn(a, b);
#else
  return a + b;
#endif
}

/* p0, p1: normal -> (c, unused); uniform -> (a, w); constant -> (a, unused). */
MOE_GEN_HD float moe_gen_value(uint64_t seed, uint32_t tensor_id, uint64_t index,
                               int dist, float p0, float p1) {
  if (dist == MOE_GEN_CONST) return p0;
  uint64_t h = moe_gen_hash(seed, tensor_id, index);
  if (dist == MOE_GEN_NORMAL) {
    int32_t s = (int32_t)(h & 0xFFFF) + (int32_t)((h >> 16) & 0xFFFF) +
                (int32_t)((h >> 32) & 0xFFFF) + (int32_t)((h >> 48) & 0xFFFF) - 131070;
    return moe_gen_mul((float)s, p0);
  }
  /* uniform */
  float t = (float)(uint32_t)(h >> 40) * (1.0f / 16777216.0f); /* exact */
  return moe_gen_add(p0, moe_gen_mul(p1, t));
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs only). */
MOE_GEN_HD uint16_t moe_gen_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#endif /* MOE_INPUTS_GEN_H */
