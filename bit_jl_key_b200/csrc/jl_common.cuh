// jl_common.cuh -- internal helpers shared by the libjlkey kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <cuda.h>

#include "jlkey.h"

namespace jlk {

// Device error word (one per device, defined in api.cu).  Kernels never trap:
// a kernel that detects a fault (a bounded wait that ran out, an impossible
// index) records a code through the pointer it was given (first fault wins)
// and returns early.  device_error_ptr() is the word's device address for the
// current device.
int *device_error_ptr();
// Unique id of the CUDA context bound to the calling thread (0 if none is
// bound yet or the driver cannot tell).  Caches of device addresses are keyed
// by it, so a context torn down and created again (cudaDeviceReset) makes
// them look the address up again instead of handing out a stale one.
unsigned long long current_context_id();

enum DeviceErr : int {
  DERR_NONE = 0,
  DERR_TC_WAIT_TIMEOUT = JL_DERR_TC_WAIT_TIMEOUT,  // tensor-core kernel: a pipeline wait ran out
  DERR_TC_TMEM_ALLOC = 2,                          // tensor-core kernel: TMEM allocation failed
  DERR_DECODE_PLAN = JL_DERR_DECODE_PLAN,          // decode: inconsistent work split
  DERR_DECODE_WAIT_TIMEOUT = JL_DERR_DECODE_WAIT_TIMEOUT,  // decode: a copy wait ran out
  DERR_INDEX = JL_DERR_INDEX,   // debug builds: an index left its buffer's extent
};

// Upper bound of every spin-wait in the library's kernels (GPU time).
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

// Test hook set by jl_test_drop_copies (host side, api.cu): when on, the
// tensor-core quantizer and the contiguous decode scorer launch without
// issuing any copy, so their consumers' waits run out after
// wait_limit_ns(); the kernels must then record the timeout, drain, free
// tensor memory and return.  Off (the default) changes nothing.
bool test_drop_copies();
unsigned long long wait_limit_ns();

__device__ __forceinline__ void record_device_error(int *err, int code) {
  atomicCAS(err, 0, code);
}

// Index checks of the debug build (compiled with -DJL_DEBUG_INDEX, which
// `python -m bit_jl_key_b200.build --debug-index` does into
// libjlkey_debug.so).  JL_IN_RANGE(err, first, count, extent) is true when
// the elements [first, first + count) lie inside a buffer of `extent`
// elements, the extent the call's shapes give that buffer; otherwise the
// debug build records DERR_INDEX in the device error word and the caller
// skips the access.  In the normal build it is the constant true and costs
// nothing.
#ifdef JL_DEBUG_INDEX
__device__ __forceinline__ bool index_in_range(int *err, int64_t first, int64_t count,
                                               int64_t extent) {
  if (first >= 0 && count >= 0 && first + count <= extent) return true;
  record_device_error(err, DERR_INDEX);
  return false;
}
#define JL_IN_RANGE(err, first, count, extent)                                   \
  ::jlk::index_in_range((err), (int64_t)(first), (int64_t)(count), (int64_t)(extent))
#else
#define JL_IN_RANGE(err, first, count, extent) true
#endif

// Number of SMs of the current device (cached per device, thread-safe).
int device_sm_count();
// Max dynamic shared memory per block (opt-in) of the current device.
int device_max_smem_optin();

// ---------------------------------------------------------------------------
// bf16 helpers on raw bit patterns.
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}
// Pack two floats into a bf16x2 register (lo -> bits 0..15), round to nearest.
// a0 += lo(w)^2 and a1 += hi(w)^2 for the two bf16 halves of w: one fma
// with bf16 multiplicands and an fp32 addend each (exactly fmaf of the
// widened halves; the widening is folded into the instruction)
__device__ __forceinline__ void bf16x2_sq_acc(uint32_t w, float &a0, float &a1) {
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n"
      " fma.rn.f32.bf16 %0, l, l, %0;\n fma.rn.f32.bf16 %1, h, h, %1;\n}\n"
      : "+f"(a0), "+f"(a1)
      : "r"(w));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_round_f32(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// ---------------------------------------------------------------------------
// PTX wrappers (sm_80+ instructions that sm_100a keeps).
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared, L2 only; src_bytes < 16 zero-fills.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src,
                                            int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst),
               "l"(src), "r"(src_bytes)
               : "memory");
}
// 8-byte async copy global -> shared; src_bytes < 8 zero-fills.
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void *src,
                                           int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(dst),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0,
                                               uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x32] * B[32x8], int8 inputs, exact int32 accumulate.
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four transposed 8x8 b16 matrices from shared memory.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0,
                                                  uint32_t &r1, uint32_t &r2,
                                                  uint32_t &r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr));
}

// ---------------------------------------------------------------------------
// mbarrier, bulk-tensor copies (TMA, never multicast) and the global timer.
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
// Arrive on `bar` once this thread's earlier cp.async copies have landed
// (the pending count is raised now and lowered by the asynchronous arrive).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}
// Wait for phase `parity` of `bar` for at most limit_ns of GPU time; false if
// the wait ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns = WAIT_LIMIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && globaltimer() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map,
                                            int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map,
                                            int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before its predecessor ends; griddep_wait() blocks
// until the predecessor has completed and its writes are visible, and
// griddep_launch_dependents() lets the next kernel start early.  Both are
// no-ops for kernels launched the ordinary way.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Host: the driver's cuTensorMapEncodeTiled (through the runtime's entry
// point query, so the library does not link libcuda); null if unavailable.
void *tensor_map_encoder();

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace jlk
