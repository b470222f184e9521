// quantize_tc.cu -- QJL key codes on the 5th-generation tensor cores.
//
// Quantizer Q(k) = sign(S k) of "The Geometry of Forgetting: How Three Papers
// Cracked KV Cache Quantization", section "QJL: one bit, zero parameters,
// unbiased inner products", for a tile of 128 keys at a time, plus the key
// norm kept beside the code (same page, "PolarQuant" section).
//
// The projection P = K S^T (M = 128 keys, N = m sketch rows, K = d) is a
// dense bf16 contraction: tcgen05.mma with both operands in shared memory
// (TMA-loaded, 128-byte swizzle, K-major) and the fp32 accumulator in tensor
// memory.  Only the sign of each accumulator element survives, so P never
// leaves the SM.
//
// One persistent CTA per SM, 10 warps with fixed roles:
//   warp 0     TMA producer: S once, then one 128 x d key tile per stage of
//              a STAGES-deep shared-memory ring.
//   warp 1     owns the TMEM allocation; one elected lane issues the MMAs
//              of each work item (a tile, or half of one at m = 512) into one
//              of two TMEM accumulators and commits them to the barriers that
//              free the key stage and publish the accumulator.
//   warps 2-5  sign epilogue: warp w reads TMEM lanes 32*(w%4).. (its lane
//              quadrant), 32 columns per tcgen05.ld, and packs the 32 sign
//              bits of a word with one funnel shift per value; then releases
//              the accumulator and stores the code row.
//   warps 6-9  norm epilogue: each thread sums the squares of one key row
//              straight from the swizzled stage in shared memory, then frees
//              the stage (together with the MMA commit).
// Every mbarrier wait is bounded (about 2 s of GPU time); a wait that runs
// out records DERR_TC_WAIT_TIMEOUT in the device error word, tells the other
// roles to stop, and the CTA still drains its copies and frees its TMEM.
#include "jl_common.cuh"
#include "jl_internal.h"
#include "jl_tc.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace jlk {
namespace tc {

constexpr int BM = 128;           // keys per tile (MMA M)
// Sign-epilogue warps per TMEM lane quadrant: 0 = chosen per shape.
#ifndef JL_QTC_SIGN_WARPS
#define JL_QTC_SIGN_WARPS 0
#endif
constexpr int SMEM_BUDGET = 220 * 1024;

template <int M, int D>
struct Cfg {
  // two sign warps per quadrant when the epilogue has many columns per byte
  // of key read (m >= 4 d) or a single accumulator (m = 512)
  static constexpr int SQ = JL_QTC_SIGN_WARPS ? JL_QTC_SIGN_WARPS
                                              : ((M >= 4 * D || M > 256) ? 2 : 1);
  static constexpr int NWARPS = 2 + 4 * SQ + 4;
  static constexpr int THREADS = NWARPS * 32;
  static constexpr int FIRST_NORM_WARP = 2 + 4 * SQ;
  static constexpr int KCH = D / 64;                 // 128-byte swizzle columns
  static constexpr int A_CHUNK = BM * 128;           // one swizzle column of a tile
  static constexpr int A_STAGE = BM * D * 2;
  static constexpr int S_CHUNK = M * 128;
  static constexpr int S_BYTES = M * D * 2;
  static constexpr int NH = (M > 256) ? 2 : 1;       // N halves (work items) per tile
  static constexpr int NMMA = M / NH;                // N of one MMA (<= 256)
  static constexpr int ACC = 2;                      // accumulator buffers (items)
  static constexpr int TMEM_COLS = ACC * NMMA;
  static constexpr int WORDS_ITEM = NMMA / 32;       // code words per item
  static constexpr int STAGES_RAW = (SMEM_BUDGET - S_BYTES) / A_STAGE;
  static constexpr int STAGES = STAGES_RAW > 6 ? 6 : STAGES_RAW;
  static constexpr int WORDS = M / 32;
  // dynamic smem: [S][A stages][barriers]
  static constexpr int OFF_A = S_BYTES;
  static constexpr int OFF_BAR = OFF_A + STAGES * A_STAGE;
  static constexpr int NBAR = 2 * STAGES + 2 * ACC + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + align slack
  static_assert(STAGES >= 2, "key ring needs two stages");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "tmem");
};

struct Params {
  int64_t n;
  int64_t num_tiles;
  uint32_t *signs;
  uint16_t *norms;
  int *err;
  unsigned long long wait_ns;  // bound of every wait (WAIT_LIMIT_NS unless a test set one)
  int drop_copies;             // test hook: issue no copy (every wait then runs out)
};

using namespace tcx;

// --------------------------------------------------------------------------
template <int M, int D>
__global__ void __launch_bounds__(Cfg<M, D>::THREADS, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_s,
                       const Params p) {
  using C = Cfg<M, D>;
  extern __shared__ uint8_t tc_smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw = smem_u32(tc_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = tc_smem_raw + (base - raw);
  const uint32_t sS = base;
  const uint32_t sA = base + C::OFF_A;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + C::ACC + a); };
  const uint32_t sfull_bar = bar0 + 8u * (2 * C::STAGES + 2 * C::ACC);
  uint32_t *tmem_holder =
      reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int *abort_flag =
      reinterpret_cast<volatile int *>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1 + 4);   // MMA commit + 4 norm warps
    }
    for (int a = 0; a < C::ACC; ++a) {
      mbar_init(tfull_bar(a), 1);       // MMA commit
      mbar_init(tempty_bar(a), 4 * C::SQ);  // the sign warps
    }
    mbar_init(sfull_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
        "tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::"r"(
            smem_u32(tmem_holder)),
        "n"(C::TMEM_COLS)
        : "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int64_t ntiles = p.num_tiles;
  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0 && !p.drop_copies) {
      mbar_expect_tx(sfull_bar, C::S_BYTES);
      for (int kc = 0; kc < C::KCH; ++kc)
        for (int h = 0; h < C::NH; ++h)
          tma_load_2d(sS + kc * C::S_CHUNK + h * C::NMMA * 128, &tmap_s, kc * 64,
                      h * C::NMMA, sfull_bar);
      int64_t i = 0;
      int s = 0;          // stage of tile i and the phase it completes next
      uint32_t ph = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
        if (!wait_phase(empty_bar(s), ph ^ 1u, abort_flag, p.err, p.wait_ns)) break;
        mbar_expect_tx(full_bar(s), C::A_STAGE);
        for (int kc = 0; kc < C::KCH; ++kc)
          tma_load_2d(sA + s * C::A_STAGE + kc * C::A_CHUNK, &tmap_k, kc * 64,
                      (int)(tile * BM), full_bar(s));
        if (++s == C::STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      // drain: the last stages issued must have landed before the CTA exits
      const int64_t issued = i;
      for (int64_t j = (issued > C::STAGES ? issued - C::STAGES : 0); j < issued; ++j) {
        const int s = (int)(j % C::STAGES);
        const uint32_t ph = (uint32_t)((j / C::STAGES) & 1);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(full_bar(s), ph) && globaltimer() - t0 < p.wait_ns) {
        }
      }
      {
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(sfull_bar, 0) && globaltimer() - t0 < p.wait_ns) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop (its waits and
    // counters stay warp-uniform) and one elected lane issues the MMAs and
    // commits.  The operand descriptors differ only in their start address
    // (bits 0-13 of the low word, address / 16), and every operand lies below
    // 256 KB of shared memory: an operand is the base descriptor plus one
    // 32-bit add.  This warp shares its sub-partition with epilogue warps
    // that keep the integer pipe busy, so its per-tile integer work is kept
    // to a few instructions.
    {
      constexpr uint32_t idesc = (1u << 4)                 // D: fp32
                                 | (1u << 7) | (1u << 10)  // A, B: bf16
                                 | ((uint32_t)(C::NMMA >> 3) << 17)  // N
                                 | ((uint32_t)(BM >> 4) << 24);      // M
      const uint64_t a0 = desc_sw128(sA), b0 = desc_sw128(sS);
      const uint32_t a_hi = (uint32_t)(a0 >> 32), a_lo0 = (uint32_t)a0;
      const uint32_t b_hi = (uint32_t)(b0 >> 32), b_lo0 = (uint32_t)b0;
      bool ok = __all_sync(0xffffffffu, wait_phase(sfull_bar, 0, abort_flag, p.err, p.wait_ns));
      int s = 0;
      uint32_t ph = 0;
      uint32_t j = 0;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        if (!__all_sync(0xffffffffu, wait_phase(full_bar(s), ph, abort_flag, p.err, p.wait_ns)))
          break;
        const uint32_t a_lo = a_lo0 + (uint32_t)s * (uint32_t)(C::A_STAGE >> 4);
#pragma unroll
        for (int h = 0; h < C::NH; ++h) {
          const uint32_t a = j & 1u;
          const uint32_t aph = (j >> 1) & 1u;
          if (!__all_sync(0xffffffffu,
                          wait_phase(tempty_bar((int)a), aph ^ 1u, abort_flag, p.err, p.wait_ns))) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t tmem_d = tmem_base + a * (uint32_t)C::NMMA;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (uint32_t)(kk & 3) * 32u;
              const uint32_t aoff = ((uint32_t)(kk >> 2) * C::A_CHUNK + koff) >> 4;
              const uint32_t boff =
                  ((uint32_t)(kk >> 2) * C::S_CHUNK + (uint32_t)h * C::NMMA * 128u + koff) >> 4;
              const uint64_t adesc = ((uint64_t)a_hi << 32) | (uint64_t)(a_lo + aoff);
              const uint64_t bdesc = ((uint64_t)b_hi << 32) | (uint64_t)(b_lo0 + boff);
              mma_ss(tmem_d, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            }
            commit(tfull_bar((int)a));
          }
          __syncwarp();
          ++j;
        }
        if (!ok) break;
        if (elect_one()) commit(empty_bar(s));
        __syncwarp();
        if (++s == C::STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (j > 0 && lane == 0) {
        const uint32_t jl = j - 1;
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(tfull_bar((int)(jl & 1)), (jl >> 1) & 1) &&
               globaltimer() - t0 < p.wait_ns) {
        }
      }
      __syncwarp();
    }
  } else if (warp < C::FIRST_NORM_WARP) {
    // ---------------- sign epilogue: TMEM lane quadrant warp % 4, and the
    // k-th of the quadrant's SQ shares of each item's code words
    const int q = warp & 3;
    const int k = (warp - 2) >> 2;
    constexpr int WPW = C::WORDS_ITEM / C::SQ;  // code words per sign warp and item
    constexpr int GW = WPW < 4 ? WPW : 4;       // words per 16/8/4-byte store
    int64_t j = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      const int64_t row = tile * BM + 32 * q + lane;
      const bool live = row < p.n;
      for (int h = 0; h < C::NH; ++h, ++j) {
        const int a = (int)(j & 1);
        const uint32_t aph = (uint32_t)((j >> 1) & 1);
        // the lanes decide together (the tensor-memory loads are warp-wide)
        if (!__all_sync(0xffffffffu, wait_phase(tfull_bar(a), aph, abort_flag, p.err, p.wait_ns))) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t trow = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * C::NMMA);
        uint32_t *dst = p.signs + row * C::WORDS + h * C::WORDS_ITEM + k * WPW;
        // this warp's WPW code words; the TMEM loads are double-buffered so
        // that the load of word w + 1 is in flight while word w is packed
        uint32_t words[WPW];
        uint32_t va[32], vb[32];
        const uint32_t tcol = trow + 32 * (k * WPW);
        ld32(tcol, va);
#pragma unroll
        for (int w = 0; w < WPW; w += 2) {
          ld_wait(va);
          if (w + 1 < WPW) ld32(tcol + 32 * (w + 1), vb);
          words[w] = sign_word(va);
          if (w + 1 < WPW) {
            ld_wait(vb);
            if (w + 2 < WPW) ld32(tcol + 32 * (w + 2), va);
            words[w + 1] = sign_word(vb);
          }
        }
        if (live && JL_IN_RANGE(p.err, row * C::WORDS + h * C::WORDS_ITEM + k * WPW, WPW,
                                p.n * C::WORDS)) {
#pragma unroll
          for (int w = 0; w < WPW; w += GW) {
            if constexpr (GW == 1)
              dst[w] = words[w];
            else if constexpr (GW == 2)
              *reinterpret_cast<uint2 *>(dst + w) = make_uint2(words[w], words[w + 1]);
            else
              *reinterpret_cast<uint4 *>(dst + w) =
                  make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(a));
      }
    }
  } else {
    // ---------------- norm epilogue: rows 32*(warp-6) .. +31 of each tile
    const int r = 32 * (warp - C::FIRST_NORM_WARP) + lane;
    int s = 0;            // stage of this tile and the phase it completes next
    uint32_t ph = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, wait_phase(full_bar(s), ph, abort_flag, p.err, p.wait_ns)))
        break;
      float ss0 = 0.f, ss1 = 0.f;
      const uint8_t *rowp = gbase + C::OFF_A + s * C::A_STAGE + r * 128;
#pragma unroll
      for (int kc = 0; kc < C::KCH; ++kc) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4 *>(
              rowp + kc * C::A_CHUNK + ((c ^ (r & 7)) << 4));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) bf16x2_sq_acc(w4[e], ss0, ss1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
      const int64_t row = tile * BM + r;
      if (row < p.n && JL_IN_RANGE(p.err, row, 1, p.n))
        p.norms[row] = __half_as_ushort(__float2half_rn(sqrtf(ss0 + ss1)));
      if (++s == C::STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem_base),
                 "n"(C::TMEM_COLS)
                 : "memory");
  }
}

// --------------------------------------------------------------------------
// host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

// 2-D bf16 tensor [rows][cols] with row pitch `pitch_elems`, boxes of
// 64 columns (128 B) x box_rows rows, 128-byte swizzle, zero fill out of range.
bool make_map(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols,
              uint64_t pitch_elems, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int M, int D>
cudaError_t launch_t(const uint16_t *K, int64_t n, int64_t ldk, const uint16_t *S,
                     uint32_t *signs, uint16_t *norms, cudaStream_t stream) {
  using C = Cfg<M, D>;
  CUtensorMap mk, ms;
  if (!make_map(&mk, K, (uint64_t)n, D, (uint64_t)ldk, BM)) return cudaErrorInvalidValue;
  if (!make_map(&ms, S, M, D, D, (uint32_t)C::NMMA)) return cudaErrorInvalidValue;
  int *err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  Params p{n, (n + BM - 1) / BM, signs, norms, err, wait_limit_ns(),
           test_drop_copies() ? 1 : 0};
  cudaError_t e = cudaFuncSetAttribute(quantize_tc_kernel<M, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.num_tiles < device_sm_count() ? p.num_tiles : device_sm_count();
  quantize_tc_kernel<M, D><<<(int)grid, C::THREADS, C::SMEM, stream>>>(mk, ms, p);
  return cudaGetLastError();
}

}  // namespace tc

bool quantize_tc_supported(int m, int d, int64_t n, int64_t ldk, const void *K) {
  if (!((d == 64 || d == 128) && (m == 64 || m == 128 || m == 256 || m == 512)))
    return false;
  if (n < 1 || n >= ((int64_t)1 << 31)) return false;  // tensor-map row extent
  if ((reinterpret_cast<uintptr_t>(K) & 15u) != 0 || ((ldk * 2) & 15) != 0) return false;
  if (ldk >= ((int64_t)1 << 39)) return false;
  return tc::encode_fn() != nullptr;
}

cudaError_t launch_quantize_tc(const uint16_t *K, int64_t n, int64_t ldk,
                               const uint16_t *S, int m, int d, uint32_t *signs,
                               uint16_t *norms, cudaStream_t stream) {
#define JL_CASE(MM, DD) \
  if (m == MM && d == DD) return tc::launch_t<MM, DD>(K, n, ldk, S, signs, norms, stream);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
