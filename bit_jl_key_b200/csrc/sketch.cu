// sketch.cu -- the seeded Gaussian sketch S (m x d, bf16).
//
// "The Geometry of Forgetting: How Three Papers Cracked KV Cache
// Quantization", section "QJL: one bit, zero parameters, unbiased inner
// products": S has i.i.d. standard normal entries and is rebuilt from a seed
// instead of being stored.  The generator is fixed by this library's ABI
// (include/jlkey.h): SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) in its
// counter form, a uniform from the top 52 bits plus half a step, the
// Box-Muller transform (cosine branch) in float64, then bf16 rounding to
// nearest-even straight from float64.
#include "jl_common.cuh"
#include "jl_internal.h"

#include <math.h>

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

__global__ void sketch_kernel(uint16_t *__restrict__ S, int64_t total,
                              uint64_t seed) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const double u1 = open_uniform(splitmix64_at(seed, 2ull * (uint64_t)e));
    const double u2 = open_uniform(splitmix64_at(seed, 2ull * (uint64_t)e + 1ull));
    const double g = sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
    S[e] = bf16_from_f64_bits(g);
  }
}

cudaError_t launch_sketch(uint16_t *S, int m, int d, uint64_t seed,
                          cudaStream_t stream) {
  const int64_t total = (int64_t)m * d;
  const int threads = 256;
  const int blocks = (int)((total + threads - 1) / threads);
  sketch_kernel<<<blocks, threads, 0, stream>>>(S, total, seed);
  return cudaGetLastError();
}

}  // namespace jlk

extern "C" uint16_t jl_bf16_from_f64(double x) {
  return jlk::bf16_from_f64_bits(x);
}
