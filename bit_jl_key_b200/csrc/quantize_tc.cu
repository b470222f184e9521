// quantize_tc.cu -- tensor-core (tcgen05 + TMA) QJL quantizer for bf16 keys.
#include "jl_common.cuh"
#include "jl_internal.h"

namespace jlk {

bool quantize_tc_supported(int m, int d, int64_t ldk, const void *K) {
  (void)m; (void)d; (void)ldk; (void)K;
  return false;
}

cudaError_t launch_quantize_tc(const uint16_t *K, int64_t n, int64_t ldk,
                               const uint16_t *S, int m, int d,
                               uint32_t *signs, uint16_t *norms,
                               cudaStream_t stream) {
  (void)K; (void)n; (void)ldk; (void)S; (void)m; (void)d; (void)signs;
  (void)norms; (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace jlk
