// decode_noalloc.cu -- decode attention for callers that cannot allocate.
//
// jl_decode_attention needs device scratch (the query projections and the
// per-split softmax states) that its caller allocates.  Some callers cannot
// allocate device memory where they call us: a plugin running inside an
// engine that owns all device memory through its own pool and hands the
// plugin no allocator, or code on a latency-critical path where cudaMalloc
// and cudaFree would stall the device.  jl_decode_attention_noalloc serves
// them: it runs the same kernels with a scratch buffer that lives in this
// file as a statically sized __device__ array, so the call allocates nothing.
//
// Costs and rules of that design:
//  - every GPU that loads the library holds JL_DECODE_STATIC_SCRATCH_BYTES
//    of device memory for the array until the process exits;
//  - all calls share the one array, so two calls whose kernels overlap on a
//    GPU (for example on two streams) race and corrupt each other's result;
//  - shapes whose scratch would exceed the array are rejected before any
//    launch;
//  - the array's device address is looked up once per device, on the first
//    call made with that device current, and looked up again only if that
//    device's context has been replaced since (cudaDeviceReset), so a reset
//    never leaves a stale address behind.
#include "jl_common.cuh"
#include "jl_internal.h"

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char
    g_decode_scratch[JL_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];

// Device address of g_decode_scratch on the current device.  In host code the
// array's name stands for a host-side shadow, not device memory, so kernels
// must be given the address the runtime reports for the current device.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = jlk::current_context_id();
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int jl_decode_attention_noalloc(
    const void *Q, jl_dtype q_dtype, const uint16_t *S, const uint32_t *signs,
    const uint16_t *norms, const uint16_t *V, int B, int Hq, int Hkv,
    int64_t T, int m, int d, float softmax_scale, uint16_t *out,
    float *scores, jl_stream_t stream) {
  // the checks of jl_decode_attention, minus the workspace
  jlk::DecodePlan p;
  bool empty = false;
  const int st = jlk::validate_decode(Q, q_dtype, S, signs, norms, V, B, Hq, Hkv, T, m, d,
                                      softmax_scale, out, scores, &p, &empty);
  if (st != JL_OK || empty) return st;
  if (p.total_bytes > (size_t)JL_DECODE_STATIC_SCRATCH_BYTES)
    return JL_ERR_SCRATCH_LIMIT;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return JL_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the kernels read only
  // elements written earlier in the same call.
  const cudaError_t e = jlk::launch_decode(p, Q, q_dtype == JL_F32, S, signs,
                                           norms, V, softmax_scale, out, scores,
                                           scratch, (cudaStream_t)stream);
  return e == cudaSuccess ? JL_OK : JL_ERR_CUDA;
}
