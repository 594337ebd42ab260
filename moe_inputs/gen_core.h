/*
 * Seeded, counter-based synthetic input generator: the per-element formulas.
 *
 * This header is the single definition of how every synthetic tensor is drawn.
 * It is included by the host implementation (gen_host.c) and by the CUDA
 * implementation (gen_cuda.cu); both produce bit-identical values because every
 * step is integer arithmetic followed by one int->float conversion and one fp32
 * multiply (both exactly rounded, no contraction possible).
 *
 * It holds none of the MoE layer's arithmetic: it only draws numbers.
 *
 *   splitmix64   : the SplitMix64 finaliser (Steele, Lea and Flood, "Fast
 *                  splittable pseudorandom number generators", OOPSLA 2014;
 *                  the constants are the published ones).
 *   key          : splitmix64(splitmix64(seed) + stream)  - one stream per tensor
 *   draw(key, i) : splitmix64(key + i)                     - random access by index
 *   normal i     : eight 16-bit fields of draw(2i) and draw(2i+1) are summed
 *                  (Irwin-Hall with 8 terms, an approximation of N(0,1) with the
 *                  exact mean 0 and variance 1 of the scaled sum, tails cut at
 *                  +-4.9 sigma);  v = 2*S - 8*65535  (even integer, |v| <= 524280)
 *                  value = (float)v * scale, scale = sigma / (65536*sqrt(8/3))
 *                  (the std of 2*S is 2*sqrt(8*(65536^2-1)/12) ~ 65536*sqrt(8/3))
 *   uniform i    : (draw(i) >> 40) * 2^-24, exactly representable, in [0, 1)
 *   bf16         : round-to-nearest-even of the fp32 value's bit pattern
 */
#ifndef MOE_INPUTS_GEN_CORE_H
#define MOE_INPUTS_GEN_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define GEN_HD __host__ __device__ __forceinline__
#else
#define GEN_HD static inline
#endif

GEN_HD uint64_t gen_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

GEN_HD uint64_t gen_key_of(uint64_t seed, uint64_t stream) {
  return gen_splitmix64(gen_splitmix64(seed) + stream);
}

GEN_HD uint64_t gen_draw(uint64_t key, uint64_t i) { return gen_splitmix64(key + i); }

/* Centred Irwin-Hall(8) integer: an even integer in [-524280, 524280]. */
GEN_HD int32_t gen_ih8(uint64_t key, uint64_t i) {
  uint64_t a = gen_draw(key, 2 * i), b = gen_draw(key, 2 * i + 1);
  int32_t s = 0;
  for (int j = 0; j < 4; ++j) {
    s += (int32_t)((a >> (16 * j)) & 0xFFFFu);
    s += (int32_t)((b >> (16 * j)) & 0xFFFFu);
  }
  return 2 * s - 8 * 65535;
}

GEN_HD float gen_normal_f32(uint64_t key, uint64_t i, float scale) {
  return (float)gen_ih8(key, i) * scale;
}

GEN_HD float gen_uniform01(uint64_t key, uint64_t i) {
  return (float)(gen_draw(key, i) >> 40) * (1.0f / 16777216.0f);
}

/* fp32 -> bf16 bit pattern, round to nearest even (NaN kept quiet). */
GEN_HD uint16_t gen_f32_to_bf16(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  uint32_t u = c.u;
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#endif
