// jl_rng.cuh -- the seeded Gaussian generator shared by the sketch and the
// rotation: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) in its counter
// form, a uniform from the top 52 bits plus half a step, the Box-Muller
// transform (cosine branch) in float64, and bf16 rounding to nearest-even
// straight from float64.
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

namespace jlk {

__host__ __device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed,
                                                           uint64_t n) {
  uint64_t z = seed + (n + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ __forceinline__ double open_uniform(uint64_t x) {
  // (j + 1/2) * 2^-52 with j the top 52 bits: strictly inside (0, 1)
  return ((double)(x >> 12) + 0.5) * 0x1p-52;
}

// float64 -> bf16 code, nearest-even, on the IEEE bit pattern.  Normal bf16
// range: add the half-ulp bias (plus the kept lsb for ties-to-even) to the
// 45 bits that are dropped; a carry moves into the exponent on its own.
// Below 2^-126 the bf16 grid is the fixed step 2^-133, rounded with rint.
__host__ __device__ inline uint16_t bf16_from_f64_bits(double x) {
  uint64_t b;
  memcpy(&b, &x, sizeof b);
  const uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  const uint64_t a = b & 0x7FFFFFFFFFFFFFFFull;
  if (a > 0x7FF0000000000000ull) return 0x7FC0;           // NaN
  const int e = (int)(a >> 52);                           // biased f64 exponent
  if (e >= 1023 - 126) {                                  // |x| >= 2^-126
    const uint64_t keep_lsb = (a >> 45) & 1ull;
    const uint64_t r = a + 0x00000FFFFFFFFFFFull + keep_lsb;
    const int er = (int)(r >> 52);
    if (er > 1023 + 127) return (uint16_t)(sign | 0x7F80u);  // overflow: inf
    return (uint16_t)(sign | ((uint32_t)(er - (1023 - 127)) << 7) |
                      (uint32_t)((r >> 45) & 0x7Full));
  }
  // subnormal bf16 (or zero): |x| * 2^133 is exact, rint rounds ties to even
  const double q = rint(fabs(x) * 0x1p133);
  return (uint16_t)(sign | (uint16_t)q);
}

// Standard normal of element e: Box-Muller (cosine branch) of the generator
// outputs 2e and 2e + 1.
__host__ __device__ __forceinline__ double gauss_at(uint64_t seed, uint64_t e) {
  const double u1 = open_uniform(splitmix64_at(seed, 2ull * e));
  const double u2 = open_uniform(splitmix64_at(seed, 2ull * e + 1ull));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

}  // namespace jlk
