// quantize_simt.cu -- QJL key codes on the SIMT cores.
//
// Quantizer Q(k) = sign(S k) ("The Geometry of Forgetting: How Three Papers
// Cracked KV Cache Quantization", section "QJL: one bit, zero parameters,
// unbiased inner products"), plus the key norm stored beside the code (same
// page, "PolarQuant" section: one radius per vector in floating point).
//
// One warp per key.  S sits transposed in shared memory (St[j][i], rows of
// M + 2 halves so that the transposing stores of consecutive columns j fall
// in different banks) so that lane l reads sketch rows 32w + l of column j
// conflict-free; lane l then
// holds (S k)_{32w + l} for every word w, and a ballot over the warp yields
// code word w directly (bit l = lane l's sign).  Products are fp32 FMA of the
// bf16 sketch with the key as stored (bf16 or fp32).
#include "jl_common.cuh"
#include "jl_internal.h"

namespace jlk {

constexpr int QS_WARPS = 8;
constexpr int QS_PAD = 2;  // halves of padding per transposed row

template <int M, int D>
constexpr int qs_smem_bytes() {
  return ((D * (M + QS_PAD) * 2 + 15) / 16) * 16 + QS_WARPS * D * 4;
}

template <int M, int D, bool F32>
__global__ void __launch_bounds__(QS_WARPS * 32)
    quantize_simt_kernel(const void *__restrict__ K, int64_t n, int64_t ldk,
                         const uint16_t *__restrict__ S,
                         uint32_t *__restrict__ signs,
                         uint16_t *__restrict__ norms, int *err) {
  // extents the shapes give the buffers (debug index checks)
  const int64_t k_extent = (n - 1) * ldk + D, s_extent = (int64_t)M * D;
  constexpr int LDT = M + QS_PAD;  // transposed row pitch (halves)
  extern __shared__ __align__(16) uint8_t qsmem[];
  uint16_t *St = reinterpret_cast<uint16_t *>(qsmem);  // [D][LDT]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float *kbuf =
      reinterpret_cast<float *>(qsmem + ((D * LDT * 2 + 15) / 16) * 16) + wid * D;
  for (int e = threadIdx.x; e < M * D; e += blockDim.x) {
    const int i = e / D, j = e - i * D;
    St[j * LDT + i] = JL_IN_RANGE(err, e, 1, s_extent) ? S[e] : (uint16_t)0;
  }
  __syncthreads();
  constexpr int WORDS = M / 32;
  for (int64_t key = (int64_t)blockIdx.x * QS_WARPS + wid; key < n;
       key += (int64_t)gridDim.x * QS_WARPS) {
    float ss = 0.f;
    for (int j = lane; j < D; j += 32) {
      const int64_t ki = key * ldk + j;
      const float v =
          !JL_IN_RANGE(err, ki, 1, k_extent) ? 0.f
          : F32 ? reinterpret_cast<const float *>(K)[ki]
                : bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(K)[ki]);
      kbuf[j] = v;
      ss = fmaf(v, v, ss);
    }
    __syncwarp();
    float acc[WORDS];
#pragma unroll
    for (int w = 0; w < WORDS; ++w) acc[w] = 0.f;
#pragma unroll 4
    for (int j = 0; j < D; ++j) {
      const float kv = kbuf[j];
#pragma unroll
      for (int w = 0; w < WORDS; ++w)
        acc[w] = fmaf(bf16_bits_to_f32(St[j * LDT + 32 * w + lane]), kv, acc[w]);
    }
#pragma unroll
    for (int w = 0; w < WORDS; ++w) {
      const uint32_t word = __ballot_sync(0xffffffffu, acc[w] >= 0.f);
      if (lane == w && JL_IN_RANGE(err, key * WORDS + w, 1, n * WORDS))
        signs[key * WORDS + w] = word;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0 && JL_IN_RANGE(err, key, 1, n))
      norms[key] = __half_as_ushort(__float2half_rn(sqrtf(ss)));
    __syncwarp();
  }
}

template <int M, int D>
static cudaError_t launch_qs(const void *K, bool f32, int64_t n, int64_t ldk,
                             const uint16_t *S, uint32_t *signs,
                             uint16_t *norms, cudaStream_t stream) {
  constexpr int smem = qs_smem_bytes<M, D>();
  auto kern = f32 ? quantize_simt_kernel<M, D, true> : quantize_simt_kernel<M, D, false>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int64_t blocks = (n + QS_WARPS - 1) / QS_WARPS;
  const int64_t cap = (int64_t)device_sm_count() * 8;
  if (blocks > cap) blocks = cap;
  int *err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  kern<<<(int)blocks, QS_WARPS * 32, smem, stream>>>(K, n, ldk, S, signs, norms, err);
  return cudaGetLastError();
}

cudaError_t launch_quantize_simt(const void *K, bool keys_f32, int64_t n,
                                 int64_t ldk, const uint16_t *S, int m, int d,
                                 uint32_t *signs, uint16_t *norms,
                                 cudaStream_t stream) {
#define JL_CASE(MM, DD) \
  if (m == MM && d == DD) \
    return launch_qs<MM, DD>(K, keys_f32, n, ldk, S, signs, norms, stream);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
