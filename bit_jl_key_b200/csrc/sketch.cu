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
#include "jl_rng.cuh"

#include <math.h>

namespace jlk {

__global__ void sketch_kernel(uint16_t *__restrict__ S, int64_t total,
                              uint64_t seed, int *err) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    if (JL_IN_RANGE(err, e, 1, total)) S[e] = bf16_from_f64_bits(gauss_at(seed, (uint64_t)e));
  }
}

cudaError_t launch_sketch(uint16_t *S, int m, int d, uint64_t seed,
                          cudaStream_t stream) {
  const int64_t total = (int64_t)m * d;
  const int threads = 256;
  const int blocks = (int)((total + threads - 1) / threads);
  int *err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  sketch_kernel<<<blocks, threads, 0, stream>>>(S, total, seed, err);
  return cudaGetLastError();
}

}  // namespace jlk

extern "C" uint16_t jl_bf16_from_f64(double x) {
  return jlk::bf16_from_f64_bits(x);
}
