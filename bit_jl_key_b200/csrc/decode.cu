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
//               its blocks through a 3-stage cp.async ring (codes + values),
//               scores them on tensor cores, keeps an online softmax and a
//               P.V accumulator per head, and writes one partial state per
//               unit it touched.
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
// goes from registers straight into the second MMA; V^T comes from shared
// memory through ldmatrix.trans on an XOR-swizzled tile.
#include "jl_common.cuh"
#include "jl_internal.h"

#include <math.h>

namespace jlk {

constexpr int DEC_KB = 32;      // keys per block
constexpr int DEC_WARPS = 4;    // warps per CTA (independent pipelines)
constexpr int DEC_STAGES = 3;   // blocks in the per-warp ring
constexpr int DEC_HPAD = 8;     // head slots per unit
constexpr int DEC_SM_COUNT = 148;  // B200; fixes the work split per shape

template <int M, int D>
struct DecCfg {
  static constexpr int WORDS = M / 32;                 // code words per key
  static constexpr int KEY_SIGN_BYTES = M / 8;
  static constexpr int SIGN_BYTES = DEC_KB * KEY_SIGN_BYTES;
  static constexpr int V_BYTES = DEC_KB * D * 2;
  static constexpr int STAGE_BYTES = SIGN_BYTES + V_BYTES;
  static constexpr int NC = M / 16;                    // 16-wide k slices
  static constexpr bool A_SMEM = (M > 256);            // A fragments in smem
  static constexpr int A_SMEM_BYTES = A_SMEM ? NC * 32 * 16 : 0;
  static constexpr int WARP_BYTES = DEC_STAGES * STAGE_BYTES + A_SMEM_BYTES;
  static constexpr int CTA_BYTES = DEC_WARPS * WARP_BYTES;
  static constexpr int LW = (M >= 128) ? M / 128 : 1;  // code words a lane reads
  static constexpr int SIGN_CHUNK = (M >= 128) ? 16 : 8;
  static constexpr int DT = D / 16;                    // 16-dim output tiles
  static constexpr int VCH = D / 8;                    // 16-byte chunks per row
};

struct DecParams {
  const float *U;           // [B][Hq][M]
  const uint32_t *signs;    // [B][Hkv][T][M/32]
  const uint16_t *norms;    // [B][Hkv][T]
  const uint16_t *V;        // [B][Hkv][T][D]
  float *partials;          // [units][slots][8][D + 2]
  float *scores;            // nullable [B][Hq][T]
  int *err;                 // device error word
  int64_t T, nb_u, NB;
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
template <int M, int D>
struct WarpRing {
  using C = DecCfg<M, D>;
  uint8_t *base;  // this warp's smem
  __device__ __forceinline__ uint8_t *sign(int s) const {
    return base + s * C::STAGE_BYTES;
  }
  __device__ __forceinline__ uint8_t *val(int s) const {
    return base + s * C::STAGE_BYTES + C::SIGN_BYTES;
  }
  __device__ __forceinline__ uint8_t *afrag() const {
    return base + DEC_STAGES * C::STAGE_BYTES;
  }
};

// Issue the async copies of block b into stage s; returns this lane's key norm
// (lane l holds key l of the block, 0 beyond the context).
template <int M, int D>
__device__ __forceinline__ float issue_block(const DecParams &p,
                                             const WarpRing<M, D> &ring,
                                             int64_t b, int64_t bend, int s,
                                             int lane) {
  using C = DecCfg<M, D>;
  float nrm = 0.f;
  if (b < bend) {
    const int64_t u = b / p.nb_u;
    const int64_t blk = b - u * p.nb_u;
    const int64_t kvi = u / p.HG;
    const int64_t key0 = blk * DEC_KB;
    const int nval = (int)((p.T - key0) < DEC_KB ? (p.T - key0) : DEC_KB);
    const int64_t gkey = kvi * p.T + key0;
    // codes: contiguous SIGN_BYTES for the block
    const uint8_t *sg = reinterpret_cast<const uint8_t *>(p.signs) +
                        gkey * C::KEY_SIGN_BYTES;
    const uint32_t sdst = smem_u32(ring.sign(s));
#pragma unroll
    for (int e = lane; e < C::SIGN_BYTES / C::SIGN_CHUNK; e += 32) {
      const int key = e * C::SIGN_CHUNK / C::KEY_SIGN_BYTES;
      const bool ok = key < nval;
      const void *src = ok ? (const void *)(sg + e * C::SIGN_CHUNK)
                           : (const void *)p.signs;
      if (C::SIGN_CHUNK == 16)
        cp_async_16(sdst + e * 16, src, ok ? 16 : 0);
      else
        cp_async_8(sdst + e * 8, src, ok ? 8 : 0);
    }
    // values: 32 rows of D bf16, 16-byte chunk c of row r stored at chunk
    // c ^ (r & 7) so that ldmatrix.trans reads are conflict-free
    const uint16_t *vg = p.V + gkey * D;
    const uint32_t vdst = smem_u32(ring.val(s));
#pragma unroll
    for (int e = lane; e < DEC_KB * C::VCH; e += 32) {
      const int key = e / C::VCH;
      const int c = e - key * C::VCH;
      const bool ok = key < nval;
      const void *src = ok ? (const void *)(vg + (int64_t)key * D + c * 8)
                           : (const void *)p.V;
      cp_async_16(vdst + key * (2 * D) + ((c ^ (key & 7)) << 4), src,
                  ok ? 16 : 0);
    }
    if (lane < nval) nrm = __half2float(__ushort_as_half(__ldg(p.norms + gkey + lane)));
  }
  cp_async_commit();
  return nrm;
}

template <int M, int D>
__global__ void __launch_bounds__(DEC_WARPS * 32)
    decode_scorer_kernel(const DecParams p) {
  using C = DecCfg<M, D>;
  extern __shared__ __align__(128) uint8_t dsmem[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int w = blockIdx.x * DEC_WARPS + wid;
  if (w >= p.W) return;
  const int g = lane >> 2;  // group id: head row / key column / dim row
  const int t = lane & 3;   // thread in group
  WarpRing<M, D> ring{dsmem + wid * C::WARP_BYTES};

  const int64_t bbeg = (int64_t)w * p.NB / p.W;
  const int64_t bend = (int64_t)(w + 1) * p.NB / p.W;

  // prologue: fill the ring
  float nrm[DEC_STAGES];
#pragma unroll
  for (int s = 0; s < DEC_STAGES; ++s)
    nrm[s] = issue_block<M, D>(p, ring, bbeg + s, bend, s, lane);

  // per-unit state
  int64_t cur_u = -1;
  int Gg = 0, b_idx = 0, hq0 = 0;
  float mx = -INFINITY, lsum = 0.f;
  float acc[C::DT][4];
  uint32_t afr[C::A_SMEM ? 1 : C::NC][4];

  auto flush = [&](int64_t u) {
    float l = lsum;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int f = warp_of_block(u * p.nb_u, p.NB, p.W);
    const int slot = w - f;
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

  for (int64_t b = bbeg; b < bend; ++b) {
    const int s = (int)((b - bbeg) % DEC_STAGES);
    const int64_t u = b / p.nb_u;
    const int64_t key0 = (b - u * p.nb_u) * DEC_KB;
    const int nval = (int)((p.T - key0) < DEC_KB ? (p.T - key0) : DEC_KB);

    if (u != cur_u) {
      if (cur_u >= 0) flush(cur_u);
      cur_u = u;
      const int64_t kvi = u / p.HG;
      const int hg = (int)(u - kvi * p.HG);
      const int hkv = (int)(kvi % p.Hkv);
      b_idx = (int)(kvi / p.Hkv);
      hq0 = hkv * p.G + hg * DEC_HPAD;
      Gg = min(DEC_HPAD, p.G - hg * DEC_HPAD);
      mx = -INFINITY;
      lsum = 0.f;
#pragma unroll
      for (int dt = 0; dt < C::DT; ++dt)
        acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
      // A fragments: rows 0..7 bf16(u), rows 8..15 bf16(u - bf16(u))
      const float *urow = p.U + ((int64_t)b_idx * p.Hq + hq0 + g) * M;
      const bool live = g < Gg;
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
          reinterpret_cast<uint4 *>(ring.afrag())[c * 32 + lane] =
              make_uint4(a4[0], a4[1], a4[2], a4[3]);
        } else {
          afr[c][0] = a4[0]; afr[c][1] = a4[1];
          afr[c][2] = a4[2]; afr[c][3] = a4[3];
        }
      }
      if constexpr (C::A_SMEM) __syncwarp();
    }

    cp_async_wait<DEC_STAGES - 1>();
    __syncwarp();

    // ---- scores for the 4 groups of 8 keys
    const uint8_t *sg = ring.sign(s);
    uint32_t wd[4][C::LW];
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) {
      const uint8_t *kp = sg + (kg * 8 + g) * C::KEY_SIGN_BYTES;
      if constexpr (M >= 128) {
#pragma unroll
        for (int i = 0; i < C::LW; ++i)
          wd[kg][i] = reinterpret_cast<const uint32_t *>(kp)[t * C::LW + i];
      } else {
        wd[kg][0] = reinterpret_cast<const uint32_t *>(kp)[t >> 1];
      }
    }
    float sc[4][4];
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) sc[kg][0] = sc[kg][1] = sc[kg][2] = sc[kg][3] = 0.f;
    const int pbase = (M >= 128) ? 0 : 8 * (t & 1);
#pragma unroll
    for (int c = 0; c < C::NC; ++c) {
      uint32_t a0, a1, a2, a3;
      if constexpr (C::A_SMEM) {
        const uint4 v = reinterpret_cast<const uint4 *>(ring.afrag())[c * 32 + lane];
        a0 = v.x; a1 = v.y; a2 = v.z; a3 = v.w;
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

    // ---- estimator, masking, online softmax (head g, keys kg*8 + 2t + j)
    float l2[4][2];
    float bmax = -INFINITY;
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = kg * 8 + 2 * t + j;
        const float raw = sc[kg][j] + sc[kg][j + 2];
        const float nk = __shfl_sync(0xffffffffu, nrm[0], key);
        const float sval = p.coef * nk * raw;
        const bool ok = key < nval;
        if (p.scores != nullptr && ok && g < Gg)
          p.scores[((int64_t)b_idx * p.Hq + hq0 + g) * p.T + key0 + key] = sval;
        l2[kg][j] = ok ? sval * p.scale_log2 : -INFINITY;
        bmax = fmaxf(bmax, l2[kg][j]);
      }
    }
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

    // ---- P.V: two k-steps of 16 keys
    const uint32_t vbase = smem_u32(ring.val(s));
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const uint32_t pb0 = pack_bf16x2(pr[2 * jj][0], pr[2 * jj][1]);
      const uint32_t pb1 = pack_bf16x2(pr[2 * jj + 1][0], pr[2 * jj + 1][1]);
      const int key = 16 * jj + rr + 8 * (mi >> 1);
#pragma unroll
      for (int dt = 0; dt < C::DT; ++dt) {
        const int ch = 2 * dt + (mi & 1);
        const uint32_t addr = vbase + key * (2 * D) + ((ch ^ rr) << 4);
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(addr, v0, v1, v2, v3);
        mma_bf16_16816(acc[dt], v0, v1, v2, v3, pb0, pb1);
      }
    }

    // ---- refill this stage with block b + STAGES
    __syncwarp();
#pragma unroll
    for (int i = 0; i < DEC_STAGES - 1; ++i) nrm[i] = nrm[i + 1];
    nrm[DEC_STAGES - 1] =
        issue_block<M, D>(p, ring, b + DEC_STAGES, bend, s, lane);
  }
  if (cur_u >= 0) flush(cur_u);
  cp_async_wait<0>();
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
template <int M, int D>
static int ctas_per_sm() {
  const int smem_sm = 228 * 1024;
  int k = smem_sm / (DecCfg<M, D>::CTA_BYTES + 1024);
  if (k > 3) k = 3;
  if (k < 1) k = 1;
  return k;
}

static int dispatch_ctas_per_sm(int m, int d) {
#define JL_CASE(MM, DD) \
  if (m == MM && d == DD) return ctas_per_sm<MM, DD>();
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return 0;
}

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool make_decode_plan(int B, int Hq, int Hkv, int64_t T, int m, int d,
                      DecodePlan *pl) {
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv) return false;
  const int k = dispatch_ctas_per_sm(m, d);
  if (k == 0) return false;
  DecodePlan p{};
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.m = m; p.d = d;
  p.G = Hq / Hkv;
  p.HG = (p.G + DEC_HPAD - 1) / DEC_HPAD;
  p.units = B * Hkv * p.HG;
  p.nb_u = (T + DEC_KB - 1) / DEC_KB;
  p.NB = (int64_t)p.units * p.nb_u;
  const int64_t wt = (int64_t)DEC_SM_COUNT * k * DEC_WARPS;
  p.W = (int)(p.NB < wt ? p.NB : wt);
  p.slots = (int)((p.W + p.units - 1) / p.units) + 1;
  p.u_bytes = round_up((size_t)B * Hq * m * sizeof(float), 256);
  p.partial_bytes = round_up(
      (size_t)p.units * p.slots * DEC_HPAD * (d + 2) * sizeof(float), 256);
  p.total_bytes = p.u_bytes + p.partial_bytes;
  *pl = p;
  return true;
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
  const int bh = pl.B * pl.Hq;
  if (q_f32)
    qproj_kernel<M, D, true><<<bh, 128, 0, stream>>>(Q, S, U);
  else
    qproj_kernel<M, D, false><<<bh, 128, 0, stream>>>(Q, S, U);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (device_error_ptr() == nullptr) return cudaErrorInvalidSymbol;

  DecParams p;
  p.U = U; p.signs = signs; p.norms = norms; p.V = V; p.partials = partials;
  p.scores = scores; p.err = device_error_ptr(); p.T = pl.T; p.nb_u = pl.nb_u; p.NB = pl.NB;
  p.Hq = pl.Hq; p.Hkv = pl.Hkv; p.G = pl.G; p.HG = pl.HG; p.W = pl.W;
  p.slots = pl.slots;
  p.coef = (float)(sqrt(M_PI / 2.0) / (double)M);
  p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634074);
  e = cudaFuncSetAttribute(decode_scorer_kernel<M, D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::CTA_BYTES);
  if (e != cudaSuccess) return e;
  const int ctas = (pl.W + DEC_WARPS - 1) / DEC_WARPS;
  decode_scorer_kernel<M, D><<<ctas, DEC_WARPS * 32, C::CTA_BYTES, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<bh, D, 0, stream>>>(partials, out, pl.Hq, pl.Hkv,
                                                 pl.G, pl.HG, pl.nb_u, pl.NB,
                                                 pl.W, pl.slots);
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
