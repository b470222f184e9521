// decode.cu -- decode attention that reads only the compressed keys.
//
// Estimator: "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with
// Zero Overhead", Abstract (QJL on the key, plain JL transform on the query),
// with the dequantizer of "The Geometry of Forgetting: How Three Papers
// Cracked KV Cache Quantization", section "QJL: one bit, zero parameters,
// unbiased inner products", taken with m sketch rows and scaled by the stored
// key norm:
//     s(q, k_t) = sqrt(pi/2)/m * ||k_t|| * sum_i (S q)_i * sign_i(k_t).
// The logits softmax_scale * s feed a softmax over the context and a sum of
// bf16 values.
//
// Three kernels on one stream:
//   1. qproj    u = S q per (b, query head), fp32.
//   2. scorer   a fixed grid of warps; the (unit, 32-key block) space is cut
//               into equal contiguous runs, one per warp.  A unit is one
//               (b, kv head, group of <= 8 query heads).  Each warp streams
//               its blocks through its own ring of shared-memory stages: one
//               lane loads the block's values with a 3-D bulk-tensor copy
//               (TMA, 128-byte swizzle, rows past the context zero-filled),
//               every lane copies a slice of the sign codes with cp.async,
//               and both complete on the stage's mbarrier.  The warp scores
//               the block on tensor cores, keeps an online softmax and a P.V
//               accumulator per head, and writes one partial state per unit
//               it touched.
//   3. combine  log-sum-exp merge of the partial states -> bf16 output.
//
// Scoring on tensor cores.  For 8 keys and one 16-wide slice of the sketch
// coordinates, D[16 x 8] += A[16 x 16] * B[16 x 8] with
//   A rows 0..7  = bf16(u) of the <= 8 heads,  rows 8..15 = bf16(u - bf16(u))
//   B[k][key]    = +1 / -1 from the sign bit of that coordinate,
// so D[h][key] + D[h+8][key] = sum_i u_i sign_i with ~16 significant bits of u
// and exact +-1 products accumulated in fp32.  The coordinate order inside
// the contraction is free, so each lane builds a +-1 bf16x2 register from bits
// p and p+16 of one code word with a shift and one LOP3:
//   ((w << (15 - p)) & 0x80008000) ^ 0xBF80BF80.
// The score accumulator layout equals the B-operand layout of the P.V product
// D[16 dims x 8 heads] += V^T[16 dims x 16 keys] * P[16 keys x 8 heads], so P
// goes from registers straight into the second MMA; V^T comes from the
// swizzled stage through ldmatrix.trans, conflict-free.
#include "jl_common.cuh"
#include "jl_internal.h"

#include <cudaTypedefs.h>
#include <math.h>

namespace jlk {

constexpr int DEC_KB = 32;         // keys per block
constexpr int DEC_WARPS = 4;       // warps per CTA (independent pipelines)
constexpr int DEC_HPAD = 8;        // head slots per unit
constexpr int DEC_SM_COUNT = 148;  // B200 SMs: bounds the workspace per shape
constexpr int DEC_MAX_CTAS_SM = 4;
constexpr int DEC_NORM_AREA = 96;  // per stage: 40 fp16 norms (aligned superset)
#ifndef JL_DECODE_S8
#define JL_DECODE_S8 0
#endif
constexpr bool DEC_S8 = JL_DECODE_S8 != 0;  // int8 scoring MMA (else bf16)

template <int M, int D>
struct DecCfg {
  static constexpr int STAGES = 2;                     // blocks in the ring
  static constexpr int KEY_SIGN_BYTES = M / 8;
  static constexpr int SIGN_BYTES = DEC_KB * KEY_SIGN_BYTES;
  static constexpr int V_BYTES = DEC_KB * D * 2;       // 4 or 8 KB
  static constexpr int V_BOX = DEC_KB * 128;           // one 64-column box
  static constexpr int STAGE_BYTES = (V_BYTES + SIGN_BYTES + 1023) / 1024 * 1024;
  // scoring MMA: bf16 m16n8k16 (16 coordinates per slice) or s8 m16n8k32 (32)
  static constexpr int KS = DEC_S8 ? 32 : 16;
  static constexpr int NC = M / KS;                    // k slices
  static constexpr int A_REGS = 4 * NC;
  static constexpr bool A_SMEM = A_REGS > 64;          // A fragments in smem
  static constexpr int A_SMEM_BYTES = A_SMEM ? NC * 32 * 16 : 0;
  static constexpr int WARP_BYTES = STAGES * STAGE_BYTES + A_SMEM_BYTES;
  static constexpr int OFF_NORM = DEC_WARPS * WARP_BYTES;
  static constexpr int OFF_BAR = OFF_NORM + DEC_WARPS * STAGES * DEC_NORM_AREA;
  static constexpr int CTA_BYTES = OFF_BAR + DEC_WARPS * STAGES * 8 + 1024;  // + align
  static constexpr int LW = (M >= 128) ? M / 128 : 1;  // code words a lane reads
  static constexpr int SIGN_CHUNK = (M >= 128) ? 16 : 8;
  static constexpr int SIGN_CHUNKS = SIGN_BYTES / SIGN_CHUNK;  // multiple of 32
  static constexpr int DT = D / 16;                    // 16-dim output tiles
  static_assert(SIGN_CHUNKS % 32 == 0, "sign chunks per lane");
  static_assert(STAGE_BYTES % 1024 == 0 && WARP_BYTES % 1024 == 0, "swizzle atoms");
};

struct DecParams {
  const float *U;           // [B][Hq][M]
  const uint32_t *signs;    // [B][Hkv][T][M/32]
  const uint16_t *norms;    // [B][Hkv][T]
  float *partials;          // [units][slots][8][D + 2]
  float *scores;            // nullable [B][Hq][T]
  int *err;                 // device error word
  int64_t T, nb_u, NB, n_keys;
  int Hq, Hkv, G, HG, W, slots;
  float coef;               // sqrt(pi/2) / m
  float scale_log2;         // softmax_scale * log2(e)
};

// warp that owns block b when NB blocks are cut into W contiguous runs
// starting at floor(w * NB / W)
__host__ __device__ __forceinline__ int warp_of_block(int64_t b, int64_t NB,
                                                      int W) {
  return (int)(((b + 1) * (int64_t)W - 1) / NB);
}

// ---------------------------------------------------------------------------
// 1. query projection u = S q (fp32 accumulate)
template <int M, int D, bool QF32>
__global__ void __launch_bounds__(128) qproj_kernel(const void *__restrict__ Q,
                                                    const uint16_t *__restrict__ S,
                                                    float *__restrict__ U) {
  __shared__ float qs[D];
  const int bh = blockIdx.x;
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    qs[j] = QF32 ? reinterpret_cast<const float *>(Q)[(int64_t)bh * D + j]
                 : bf16_bits_to_f32(
                       reinterpret_cast<const uint16_t *>(Q)[(int64_t)bh * D + j]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    const uint4 *row = reinterpret_cast<const uint4 *>(S + (int64_t)i * D);
    float acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
      const uint4 v = __ldg(row + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(w[e] << 16), qs[c * 8 + 2 * e], acc);
        acc = fmaf(__uint_as_float(w[e] & 0xFFFF0000u), qs[c * 8 + 2 * e + 1], acc);
      }
    }
    U[(int64_t)bh * M + i] = acc;
  }
}

// ---------------------------------------------------------------------------
// 2. scorer

// Position of a block in the (unit, block) space, advanced without division.
struct BlockPos {
  int64_t u;    // unit
  int64_t blk;  // block within the unit
  __device__ __forceinline__ void next(int64_t nb_u) {
    if (++blk == nb_u) {
      blk = 0;
      ++u;
    }
  }
};

template <int M, int D>
struct Ring {
  using C = DecCfg<M, D>;
  uint32_t base;   // this warp's stages (1024-aligned)
  uint32_t nbase;  // this warp's norm areas
  uint32_t bbase;  // this warp's barriers
  __device__ __forceinline__ uint32_t val(int s) const { return base + s * C::STAGE_BYTES; }
  __device__ __forceinline__ uint32_t sign(int s) const {
    return base + s * C::STAGE_BYTES + C::V_BYTES;
  }
  __device__ __forceinline__ uint32_t afrag() const { return base + C::STAGES * C::STAGE_BYTES; }
  __device__ __forceinline__ uint32_t norm(int s) const { return nbase + s * DEC_NORM_AREA; }
  __device__ __forceinline__ uint32_t bar(int s) const { return bbase + 8 * s; }
};

// Start the copies of block `pos` into stage s: values by one 3-D bulk-tensor
// copy per 64 columns (lane 0), codes and norms by cp.async (all lanes).
template <int M, int D>
__device__ __forceinline__ void issue_block(const DecParams &p, const CUtensorMap *vmap,
                                            const Ring<M, D> &ring, const BlockPos &pos,
                                            int s, int lane) {
  using C = DecCfg<M, D>;
  const int64_t kvi = p.HG == 1 ? pos.u : pos.u / p.HG;
  const int64_t key0 = pos.blk * DEC_KB;
  const int64_t left = p.T - key0;
  const int nval = left < DEC_KB ? (int)left : DEC_KB;
  const int64_t gkey = kvi * p.T + key0;
  // codes: SIGN_BYTES contiguous bytes, a slice per lane, zero past the context
  const uint8_t *sg = reinterpret_cast<const uint8_t *>(p.signs) + gkey * C::KEY_SIGN_BYTES;
  const uint32_t sdst = ring.sign(s);
#pragma unroll
  for (int e = lane; e < C::SIGN_CHUNKS; e += 32) {
    const bool ok = e * C::SIGN_CHUNK < nval * C::KEY_SIGN_BYTES;
    const void *src = ok ? (const void *)(sg + e * C::SIGN_CHUNK) : (const void *)p.signs;
    if constexpr (C::SIGN_CHUNK == 16)
      cp_async_16(sdst + e * 16, src, ok ? 16 : 0);
    else
      cp_async_8(sdst + e * 8, src, ok ? 8 : 0);
  }
  // norms: the 16-byte-aligned run of 8-norm groups covering the block
  // (at most 5 groups); key k of the block lands at element (gkey & 7) + k
  if (lane < 5) {
    const int64_t first = (gkey & ~(int64_t)7) + 8 * lane;
    const int64_t avail = p.n_keys - first;
    const bool ok = first < gkey + nval && avail > 0;
    const int nbytes = ok ? (avail >= 8 ? 16 : (int)avail * 2) : 0;
    cp_async_16(ring.norm(s) + 16 * lane, ok ? (const void *)(p.norms + first)
                                             : (const void *)p.norms, nbytes);
  }
  cp_async_mbar_arrive(ring.bar(s));
  __syncwarp();
  if (lane == 0) {
    mbar_expect_tx(ring.bar(s), C::V_BYTES);
#pragma unroll
    for (int h = 0; h < D / 64; ++h)
      tma_load_3d(ring.val(s) + h * C::V_BOX, vmap, h * 64, (int)key0, (int)kvi, ring.bar(s));
  }
}

__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

template <int M, int D>
__global__ void __launch_bounds__(DEC_WARPS * 32)
    decode_scorer_kernel(const __grid_constant__ CUtensorMap vmap, const DecParams p) {
  using C = DecCfg<M, D>;
  extern __shared__ uint8_t dsmem_raw[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int w = blockIdx.x * DEC_WARPS + wid;
  if (w >= p.W) return;
  const int g = lane >> 2;  // group id: head row / key column / dim row
  const int t = lane & 3;   // thread in group
  const uint32_t cta = (smem_u32(dsmem_raw) + 1023u) & ~1023u;
  const Ring<M, D> ring{cta + wid * C::WARP_BYTES,
                        cta + C::OFF_NORM + wid * C::STAGES * DEC_NORM_AREA,
                        cta + C::OFF_BAR + wid * C::STAGES * 8};

  const int64_t bbeg = (int64_t)w * p.NB / p.W;
  const int64_t bend = (int64_t)(w + 1) * p.NB / p.W;
  const int64_t nblk = bend - bbeg;

  if (lane == 0)
    for (int s = 0; s < C::STAGES; ++s) mbar_init(ring.bar(s), 1);
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  __syncwarp();

  // prologue: fill the ring
  BlockPos ipos{bbeg / p.nb_u, bbeg - (bbeg / p.nb_u) * p.nb_u};
  const BlockPos pos0 = ipos;
#pragma unroll
  for (int s = 0; s < C::STAGES; ++s) {
    if (s < nblk) {
      issue_block<M, D>(p, &vmap, ring, ipos, s, lane);
      ipos.next(p.nb_u);
    }
  }

  // per-unit state
  int64_t cur_u = -1, kv_base = 0;
  int Gg = 0, b_idx = 0, hq0 = 0;
  float mx = -INFINITY, lsum = 0.f;
  float hscale = 0.f;   // int8 scoring: value of one unit of S q for head g
  int usum = 0;         // int8 scoring: sum of the quantized S q of head g
  float acc[C::DT][4];
  uint32_t afr[C::A_SMEM ? 1 : C::NC][4];
  bool failed = false;

  auto flush = [&](int64_t u) {
    float l = lsum;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int slot = w - warp_of_block(u * p.nb_u, p.NB, p.W);
    if (slot < 0 || slot >= p.slots) {
      record_device_error(p.err, DERR_DECODE_PLAN);
      return;
    }
    float *rec = p.partials + ((size_t)u * p.slots + slot) * DEC_HPAD * (D + 2);
    if (t == 0 && g < Gg) {
      rec[g * (D + 2) + D] = mx;
      rec[g * (D + 2) + D + 1] = l;
    }
    const int h0 = 2 * t, h1 = 2 * t + 1;
#pragma unroll
    for (int dt = 0; dt < C::DT; ++dt) {
      const int d0 = dt * 16 + g, d1 = d0 + 8;
      if (h0 < Gg) {
        rec[h0 * (D + 2) + d0] = acc[dt][0];
        rec[h0 * (D + 2) + d1] = acc[dt][2];
      }
      if (h1 < Gg) {
        rec[h1 * (D + 2) + d0] = acc[dt][1];
        rec[h1 * (D + 2) + d1] = acc[dt][3];
      }
    }
  };

  BlockPos pos = pos0;
  for (int64_t i = 0; i < nblk; ++i) {
    const int s = (int)(i % C::STAGES);
    const int64_t u = pos.u;
    const int64_t key0 = pos.blk * DEC_KB;
    const int64_t left = p.T - key0;
    const int nval = left < DEC_KB ? (int)left : DEC_KB;

    if (u != cur_u) {
      if (cur_u >= 0) flush(cur_u);
      cur_u = u;
      const int64_t kvi = u / p.HG;
      const int hg = (int)(u - kvi * p.HG);
      const int hkv = (int)(kvi % p.Hkv);
      kv_base = kvi * p.T;
      b_idx = (int)(kvi / p.Hkv);
      hq0 = hkv * p.G + hg * DEC_HPAD;
      Gg = min(DEC_HPAD, p.G - hg * DEC_HPAD);
      mx = -INFINITY;
      lsum = 0.f;
#pragma unroll
      for (int dt = 0; dt < C::DT; ++dt)
        acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
      const float *urow = p.U + ((int64_t)b_idx * p.Hq + hq0 + g) * M;
      const bool live = g < Gg;
      if constexpr (DEC_S8) {
        // S q of head g as integers: u ~= hscale * (256 hi + lo), |256 hi + lo|
        // <= 32000, hi and lo int8 (rows g and g + 8 of the A operand)
        float amax = 0.f;
        for (int q = 0; q < M / 16; ++q) {
          const int Qr = t * (M / 16) + q;
          const int ib = 32 * (Qr >> 3) + (Qr & 7);
#pragma unroll
          for (int j = 0; j < 4; ++j) amax = fmaxf(amax, live ? fabsf(urow[ib + 8 * j]) : 0.f);
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        hscale = amax > 0.f ? amax / 32000.f : 0.f;
        const float inv = amax > 0.f ? 32000.f / amax : 0.f;
        int lsum_i = 0;
#pragma unroll
        for (int c = 0; c < C::NC; ++c) {
          uint32_t a4[4];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int Qr = t * (M / 16) + 2 * c + r;  // byte-register index in the code
            const int ib = 32 * (Qr >> 3) + (Qr & 7);
            int hi[4], lo[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int ui = live ? __float2int_rn(urow[ib + 8 * j] * inv) : 0;
              lsum_i += ui;
              hi[j] = (ui + 128) >> 8;
              lo[j] = ui - (hi[j] << 8);
            }
            a4[r == 0 ? 0 : 2] = pack_s8x4(hi[0], hi[1], hi[2], hi[3]);
            a4[r == 0 ? 1 : 3] = pack_s8x4(lo[0], lo[1], lo[2], lo[3]);
          }
          if constexpr (C::A_SMEM) {
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                             ring.afrag() + (c * 32 + lane) * 16),
                         "r"(a4[0]), "r"(a4[1]), "r"(a4[2]), "r"(a4[3])
                         : "memory");
          } else {
            afr[c][0] = a4[0]; afr[c][1] = a4[1];
            afr[c][2] = a4[2]; afr[c][3] = a4[3];
          }
        }
        lsum_i += __shfl_xor_sync(0xffffffffu, lsum_i, 1);
        lsum_i += __shfl_xor_sync(0xffffffffu, lsum_i, 2);
        usum = lsum_i;
      } else {
        // A fragments: rows 0..7 bf16(u), rows 8..15 bf16(u - bf16(u))
#pragma unroll
        for (int c = 0; c < C::NC; ++c) {
          uint32_t a4[4];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int Qp = t * (M / 8) + 2 * c + r;  // pair index in the key code
            const int ilo = 32 * (Qp >> 4) + (Qp & 15);
            const float x0 = live ? urow[ilo] : 0.f;
            const float x1 = live ? urow[ilo + 16] : 0.f;
            const float h0 = bf16_round_f32(x0), h1 = bf16_round_f32(x1);
            a4[2 * r] = pack_bf16x2(h0, h1);
            a4[2 * r + 1] = pack_bf16x2(x0 - h0, x1 - h1);
          }
          if constexpr (C::A_SMEM) {
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                             ring.afrag() + (c * 32 + lane) * 16),
                         "r"(a4[0]), "r"(a4[1]), "r"(a4[2]), "r"(a4[3])
                         : "memory");
          } else {
            afr[c][0] = a4[0]; afr[c][1] = a4[1];
            afr[c][2] = a4[2]; afr[c][3] = a4[3];
          }
        }
      }
      if constexpr (C::A_SMEM) __syncwarp();
    }

    if (!mbar_wait_bounded(ring.bar(s), (uint32_t)((i / C::STAGES) & 1))) {
      record_device_error(p.err, DERR_DECODE_WAIT_TIMEOUT);
      failed = true;
      break;
    }

    // ---- code words of the 4 groups of 8 keys (lane: key kg*8 + g)
    const uint32_t sg = ring.sign(s);
    uint32_t wd[4][C::LW];
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) {
      const uint32_t kp = sg + (kg * 8 + g) * C::KEY_SIGN_BYTES;
      if constexpr (C::LW == 4) {
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                     : "=r"(wd[kg][0]), "=r"(wd[kg][1]), "=r"(wd[kg][2]), "=r"(wd[kg][3])
                     : "r"(kp + t * 16));
      } else if constexpr (C::LW == 2) {
        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];\n"
                     : "=r"(wd[kg][0]), "=r"(wd[kg][1])
                     : "r"(kp + t * 8));
      } else if constexpr (M == 128) {
        asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(wd[kg][0]) : "r"(kp + t * 4));
      } else {
        asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(wd[kg][0]) : "r"(kp + (t >> 1) * 4));
      }
    }

    // ---- raw estimator sum_i u_i sign_i for head g, keys kg*8 + 2t + j
    float raw[4][2];
    if constexpr (DEC_S8) {
      int sc[4][4];
#pragma unroll
      for (int kg = 0; kg < 4; ++kg) sc[kg][0] = sc[kg][1] = sc[kg][2] = sc[kg][3] = 0;
      const int pbase = (M >= 128) ? 0 : 4 * (t & 1);
#pragma unroll
      for (int c = 0; c < C::NC; ++c) {
        uint32_t a0, a1, a2, a3;
        if constexpr (C::A_SMEM) {
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                       : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                       : "r"(ring.afrag() + (c * 32 + lane) * 16));
        } else {
          a0 = afr[c][0]; a1 = afr[c][1]; a2 = afr[c][2]; a3 = afr[c][3];
        }
        const int q0 = 2 * c, q1 = 2 * c + 1;
#pragma unroll
        for (int kg = 0; kg < 4; ++kg) {
          uint32_t w0, w1;
          int p0, p1;
          if constexpr (M >= 128) {
            w0 = wd[kg][q0 >> 3]; p0 = q0 & 7;
            w1 = wd[kg][q1 >> 3]; p1 = q1 & 7;
          } else {
            w0 = w1 = wd[kg][0]; p0 = pbase + q0; p1 = pbase + q1;
          }
          // bytes j = bits p + 8j: {0, 1} per coordinate
          const uint32_t b0 = (w0 >> p0) & 0x01010101u;
          const uint32_t b1 = (w1 >> p1) & 0x01010101u;
          mma_s8_16832(sc[kg], a0, a1, a2, a3, b0, b1);
        }
      }
      // sum_i u_i sign_i = hscale * (2 * sum_{bit=1} u_int - sum u_int)
#pragma unroll
      for (int kg = 0; kg < 4; ++kg)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          raw[kg][j] = hscale * (float)(2 * (sc[kg][j] * 256 + sc[kg][j + 2]) - usum);
    } else {
      float sc[4][4];
#pragma unroll
      for (int kg = 0; kg < 4; ++kg) sc[kg][0] = sc[kg][1] = sc[kg][2] = sc[kg][3] = 0.f;
      const int pbase = (M >= 128) ? 0 : 8 * (t & 1);
#pragma unroll
      for (int c = 0; c < C::NC; ++c) {
        uint32_t a0, a1, a2, a3;
        if constexpr (C::A_SMEM) {
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                       : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                       : "r"(ring.afrag() + (c * 32 + lane) * 16));
        } else {
          a0 = afr[c][0]; a1 = afr[c][1]; a2 = afr[c][2]; a3 = afr[c][3];
        }
        const int q0 = 2 * c, q1 = 2 * c + 1;
#pragma unroll
        for (int kg = 0; kg < 4; ++kg) {
          uint32_t w0, w1;
          int p0, p1;
          if constexpr (M >= 128) {
            w0 = wd[kg][q0 >> 4]; p0 = q0 & 15;
            w1 = wd[kg][q1 >> 4]; p1 = q1 & 15;
          } else {
            w0 = w1 = wd[kg][0]; p0 = pbase + q0; p1 = pbase + q1;
          }
          const uint32_t b0 = ((w0 << (15 - p0)) & 0x80008000u) ^ 0xBF80BF80u;
          const uint32_t b1 = ((w1 << (15 - p1)) & 0x80008000u) ^ 0xBF80BF80u;
          mma_bf16_16816(sc[kg], a0, a1, a2, a3, b0, b1);
        }
      }
#pragma unroll
      for (int kg = 0; kg < 4; ++kg)
#pragma unroll
        for (int j = 0; j < 2; ++j) raw[kg][j] = sc[kg][j] + sc[kg][j + 2];
    }

    // ---- estimator, masking, online softmax (head g, keys kg*8 + 2t + j)
    float l2[4][2];
    float bmax = -INFINITY;
    const uint32_t nrow = ring.norm(s) + (uint32_t)((kv_base + key0) & 7) * 2;
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = kg * 8 + 2 * t + j;
        unsigned short hb;
        asm volatile("ld.shared.u16 %0, [%1];\n" : "=h"(hb) : "r"(nrow + key * 2));
        const float nk = __half2float(__ushort_as_half(hb));
        const float sval = (p.coef * nk) * raw[kg][j];
        l2[kg][j] = sval * p.scale_log2;
        if (p.scores != nullptr && key < nval && g < Gg)
          p.scores[((int64_t)b_idx * p.Hq + hq0 + g) * p.T + key0 + key] = sval;
      }
    }
    if (nval < DEC_KB) {
#pragma unroll
      for (int kg = 0; kg < 4; ++kg)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          if (kg * 8 + 2 * t + j >= nval) l2[kg][j] = -INFINITY;
    }
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) bmax = fmaxf(bmax, fmaxf(l2[kg][0], l2[kg][1]));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
    const float mnew = fmaxf(mx, bmax);
    const float alpha = fast_exp2(mx - mnew);  // 0 on the first block
    mx = mnew;
    float pr[4][2];
    float psum = 0.f;
#pragma unroll
    for (int kg = 0; kg < 4; ++kg)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        pr[kg][j] = fast_exp2(l2[kg][j] - mnew);
        psum += pr[kg][j];
      }
    lsum = lsum * alpha + psum;
    // rescale the accumulator: lane holds heads 2t and 2t+1
    const float al0 = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
    const float al1 = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
#pragma unroll
    for (int dt = 0; dt < C::DT; ++dt) {
      acc[dt][0] *= al0; acc[dt][1] *= al1;
      acc[dt][2] *= al0; acc[dt][3] *= al1;
    }

    // ---- P.V: two k-steps of 16 keys over the swizzled value tile
    const uint32_t vbase = ring.val(s);
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const uint32_t pb0 = pack_bf16x2(pr[2 * jj][0], pr[2 * jj][1]);
      const uint32_t pb1 = pack_bf16x2(pr[2 * jj + 1][0], pr[2 * jj + 1][1]);
      const uint32_t krow = vbase + (16 * jj + rr + 8 * (mi >> 1)) * 128;
#pragma unroll
      for (int dt = 0; dt < C::DT; ++dt) {
        const int ch = 2 * dt + (mi & 1);  // 16-byte chunk along d
        const uint32_t addr = krow + (ch >> 3) * C::V_BOX + (((ch & 7) ^ rr) << 4);
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(addr, v0, v1, v2, v3);
        mma_bf16_16816(acc[dt], v0, v1, v2, v3, pb0, pb1);
      }
    }

    // ---- refill this stage with the block STAGES ahead
    __syncwarp();
    if (i + C::STAGES < nblk) {
      issue_block<M, D>(p, &vmap, ring, ipos, s, lane);
      ipos.next(p.nb_u);
    }
    pos.next(p.nb_u);
  }
  if (failed) {
    // let the copies already started land before the warp's smem goes away
    for (int k = 0; k < C::STAGES; ++k) {
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(ring.bar(k), 0) && !mbar_try_wait(ring.bar(k), 1) &&
             globaltimer() - t0 < WAIT_LIMIT_NS) {
      }
    }
    return;
  }
  if (cur_u >= 0) flush(cur_u);
}

// ---------------------------------------------------------------------------
// 3. combine the partial states of each (b, query head)
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(
    const float *__restrict__ partials, uint16_t *__restrict__ out, int Hq,
    int Hkv, int G, int HG, int64_t nb_u, int64_t NB, int W, int slots) {
  const int bh = blockIdx.x;
  const int b = bh / Hq, hq = bh - b * Hq;
  const int hkv = hq / G, hl = hq - hkv * G;
  const int hg = hl / DEC_HPAD, hh = hl - hg * DEC_HPAD;
  const int64_t u = ((int64_t)b * Hkv + hkv) * HG + hg;
  const int f = warp_of_block(u * nb_u, NB, W);
  const int l = warp_of_block((u + 1) * nb_u - 1, NB, W);
  const int n = min(l - f + 1, slots);
  const float *rec0 = partials + (size_t)u * slots * DEC_HPAD * (D + 2) +
                      (size_t)hh * (D + 2);
  const size_t sstride = (size_t)DEC_HPAD * (D + 2);
  float Mx = -INFINITY;
  for (int s = 0; s < n; ++s) Mx = fmaxf(Mx, rec0[s * sstride + D]);
  float L = 0.f, o = 0.f;
  const int dim = threadIdx.x;
  for (int s = 0; s < n; ++s) {
    const float *rec = rec0 + s * sstride;
    const float wgt = fast_exp2(rec[D] - Mx);
    L = fmaf(wgt, rec[D + 1], L);
    o = fmaf(wgt, rec[dim], o);
  }
  out[(int64_t)bh * D + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(o / L));
}

// ---------------------------------------------------------------------------
// planning and launch
static bool supported(int m, int d) {
  return (d == 64 || d == 128) && (m == 64 || m == 128 || m == 256 || m == 512);
}

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool make_decode_plan(int B, int Hq, int Hkv, int64_t T, int m, int d,
                      DecodePlan *pl) {
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv) return false;
  if ((int64_t)B * Hkv >= ((int64_t)1 << 31) || T >= ((int64_t)1 << 31)) return false;
  if (!supported(m, d)) return false;
  DecodePlan p{};
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.m = m; p.d = d;
  p.G = Hq / Hkv;
  p.HG = (p.G + DEC_HPAD - 1) / DEC_HPAD;
  p.units = B * Hkv * p.HG;
  p.nb_u = (T + DEC_KB - 1) / DEC_KB;
  p.NB = (int64_t)p.units * p.nb_u;
  // the launch uses at most W_bound warps (B200 SMs x max CTAs per SM); the
  // partial-state layout is sized for that bound so that it depends on the
  // shapes only
  const int64_t wb = (int64_t)DEC_SM_COUNT * DEC_MAX_CTAS_SM * DEC_WARPS;
  p.W = (int)(p.NB < wb ? p.NB : wb);
  p.slots = (int)((p.W + p.units - 1) / p.units) + 1;
  p.u_bytes = round_up((size_t)B * Hq * m * sizeof(float), 256);
  p.partial_bytes = round_up(
      (size_t)p.units * p.slots * DEC_HPAD * (d + 2) * sizeof(float), 256);
  p.total_bytes = p.u_bytes + p.partial_bytes;
  *pl = p;
  return true;
}

// V viewed as [B*Hkv][T][d] bf16; boxes of 64 columns x 32 rows x 1 unit with
// the 128-byte swizzle; rows past T are zero-filled.
static bool make_value_map(CUtensorMap *map, const uint16_t *V, int64_t units_kv,
                           int64_t T, int d) {
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)units_kv};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)T * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)DEC_KB, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(V), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int M, int D>
static cudaError_t launch_decode_t(const DecodePlan &pl, const void *Q,
                                   bool q_f32, const uint16_t *S,
                                   const uint32_t *signs, const uint16_t *norms,
                                   const uint16_t *V, float softmax_scale,
                                   uint16_t *out, float *scores,
                                   void *workspace, cudaStream_t stream) {
  using C = DecCfg<M, D>;
  float *U = reinterpret_cast<float *>(workspace);
  float *partials =
      reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + pl.u_bytes);
  CUtensorMap vmap;
  if (!make_value_map(&vmap, V, (int64_t)pl.B * pl.Hkv, pl.T, D))
    return cudaErrorInvalidValue;
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
  const int bh = pl.B * pl.Hq;
  if (q_f32)
    qproj_kernel<M, D, true><<<bh, 128, 0, stream>>>(Q, S, U);
  else
    qproj_kernel<M, D, false><<<bh, 128, 0, stream>>>(Q, S, U);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  DecParams p;
  p.U = U; p.signs = signs; p.norms = norms; p.partials = partials;
  p.scores = scores; p.err = err; p.T = pl.T; p.nb_u = pl.nb_u; p.NB = pl.NB;
  p.n_keys = (int64_t)pl.B * pl.Hkv * pl.T;
  p.Hq = pl.Hq; p.Hkv = pl.Hkv; p.G = pl.G; p.HG = pl.HG;
  p.slots = pl.slots;
  p.coef = (float)(sqrt(M_PI / 2.0) / (double)M);
  p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634074);
  e = cudaFuncSetAttribute(decode_scorer_kernel<M, D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::CTA_BYTES);
  if (e != cudaSuccess) return e;
  // one wave of resident CTAs, never more warps than the plan's bound
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_scorer_kernel<M, D>,
                                                    DEC_WARPS * 32, C::CTA_BYTES);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  if (per_sm > DEC_MAX_CTAS_SM) per_sm = DEC_MAX_CTAS_SM;
  const int64_t wave = (int64_t)device_sm_count() * per_sm * DEC_WARPS;
  p.W = (int)(wave < pl.W ? wave : pl.W);
  const int ctas = (p.W + DEC_WARPS - 1) / DEC_WARPS;
  decode_scorer_kernel<M, D><<<ctas, DEC_WARPS * 32, C::CTA_BYTES, stream>>>(vmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<bh, D, 0, stream>>>(partials, out, pl.Hq, pl.Hkv,
                                                 pl.G, pl.HG, pl.nb_u, pl.NB,
                                                 p.W, pl.slots);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodePlan &pl, const void *Q, bool q_f32,
                          const uint16_t *S, const uint32_t *signs,
                          const uint16_t *norms, const uint16_t *V,
                          float softmax_scale, uint16_t *out, float *scores,
                          void *workspace, cudaStream_t stream) {
#define JL_CASE(MM, DD)                                                       \
  if (pl.m == MM && pl.d == DD)                                               \
    return launch_decode_t<MM, DD>(pl, Q, q_f32, S, signs, norms, V,          \
                                   softmax_scale, out, scores, workspace,     \
                                   stream);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
