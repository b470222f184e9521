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

#include <utility>

namespace jlk {

constexpr int DEC_KB = 32;         // keys per block
constexpr int DEC_WARPS = 4;       // warps per CTA (independent pipelines)
constexpr int DEC_HPAD = 8;        // head slots per unit
constexpr int DEC_SM_COUNT = 148;  // B200 SMs: bounds the workspace per shape
constexpr int DEC_MAX_CTAS_SM = 4;
constexpr int DEC_NORM_AREA = 128; // per stage: 40 fp16 norms; bulk-tensor copies need
                                   // a 128-byte-aligned destination
// Scoring MMA per shape: 0 = chosen by decode_use_s8(), 1 = bf16, 2 = int8.
#ifndef JL_DECODE_SCORE
#define JL_DECODE_SCORE 0
#endif

// TB > 0: TurboQuant-prod codes, TB cell bit planes of D bits ahead of the M
// residual sign bits.  A symmetric codebook's centroid is a sum of +-1 terms
// over the planes: one per plane for TB <= 2, and for TB = 3 the three planes
// plus their product (whose bit is the XOR of the three), so a key is scored
// as TERMS + 1 sign contractions.  The scorer contracts code words four at a
// time (128 coordinates, one integer scale per segment), so each segment --
// the plane terms' TERMS * D coordinates, then the M residual signs -- is
// padded to whole runs of 128 coordinates whose query weights are zero (at
// D = 128 nothing is padded).
template <int M, int D, int TB>
struct TurboRow {
  static constexpr int TERMS = TB == 3 ? 4 : TB;
  static constexpr int MSE = (TERMS * D + 127) / 128 * 128;  // padded plane-term segment
  static constexpr int QJL = (M + 127) / 128 * 128;          // padded residual segment
  static constexpr int LEN = MSE + QJL;                      // query row length
};

template <int M, int D, bool S8, int TB = 0>
struct DecCfg {
  static constexpr int STAGES = 2;                     // blocks in the ring
  static constexpr int TERMS = TB == 3 ? 4 : TB;       // +-1 plane terms
  // coordinates contracted per key (TurboQuant: the padded query row)
  static constexpr int CODE_BITS = TB ? TurboRow<M, D, TB>::LEN : M;
  static constexpr int MSE_RUNS = TB ? TurboRow<M, D, TB>::MSE / 128 : 0;  // plane-term runs
  static constexpr int KEY_SIGN_BYTES = (TB * D + M) / 8;  // bytes stored per key
  static constexpr int SIGN_BYTES = DEC_KB * KEY_SIGN_BYTES;
  static constexpr int V_BYTES = DEC_KB * D * 2;       // 4 or 8 KB
  static constexpr int V_BOX = DEC_KB * 128;           // one 64-column box
  static constexpr int STAGE_BYTES = (V_BYTES + SIGN_BYTES + 1023) / 1024 * 1024;
  // scoring MMA: bf16 m16n8k16 (16 coordinates per slice) or s8 m16n8k32 (32)
  static constexpr int KS = S8 ? 32 : 16;
  static constexpr int NC = CODE_BITS / KS;            // k slices
  static constexpr int NC_MSE = MSE_RUNS * 128 / KS;   // slices of the cell planes
  static constexpr int A_REGS = 4 * NC;
  // A fragments in smem when they would crowd the registers; the cell-plane
  // codes keep theirs in registers (two CTAs per SM instead of one)
  static constexpr bool A_SMEM = A_REGS > (TB ? 96 : 64);
  static constexpr int A_SMEM_BYTES = A_SMEM ? NC * 32 * 16 : 0;
  static constexpr int WARP_BYTES = STAGES * STAGE_BYTES + A_SMEM_BYTES;
  // per stage: the block's norms (TB > 0: two binary16 per key), with room
  // for the 16-byte-aligned groups of the cp.async path
  static constexpr int NORM_BYTES = TB ? 4 : 2;
  static constexpr int NORM_AREA = TB ? 2 * DEC_NORM_AREA : DEC_NORM_AREA;
  static constexpr int OFF_NORM = DEC_WARPS * WARP_BYTES;
  static constexpr int OFF_BAR = OFF_NORM + DEC_WARPS * STAGES * NORM_AREA;
  static constexpr int CTA_BYTES = OFF_BAR + DEC_WARPS * STAGES * 8 + 1024;  // + align
  static constexpr int LW = (CODE_BITS >= 128) ? CODE_BITS / 128 : 1;  // code words a lane reads
  static constexpr int SIGN_CHUNK = (M >= 128) ? 16 : 8;
  static constexpr int SIGN_CHUNKS = SIGN_BYTES / SIGN_CHUNK;  // multiple of 32
  static constexpr int DT = D / 16;                    // 16-dim output tiles
  static_assert(SIGN_CHUNKS % 32 == 0, "sign chunks per lane");
  static_assert(TB == 0 || ((D == 128 || D == 64) && M == D), "cell-plane codes: m = d = 64 or 128");
  static_assert(STAGE_BYTES % 1024 == 0 && WARP_BYTES % 1024 == 0, "swizzle atoms");
};

struct DecParams {
  const float *U;           // [B][Hq][M]
  const uint32_t *signs;    // [B][Hkv][T][M/32]
  const uint16_t *norms;    // [B][Hkv][T]
  float *partials;          // [W + units records][8][D + 2]
  float *scores;            // nullable [B][Hq][T]
  int *err;                 // device error word
  int64_t T, nb_u, NB, n_keys;
  int Hq, Hkv, G, HG, W, slots;  // slots: partial records (W bound + units)
  float coef;               // sqrt(pi/2) / m
  float scale_log2;         // softmax_scale * log2(e)
  int64_t score_stride;     // row stride of `scores` (T, or max_len when paged)
  // paged cache (PAGED kernels): sequence b holds UH = Hkv * HG consecutive
  // units, each of paged_blocks(b) blocks, so the flat block space follows
  // from seq_lens alone; the keys live in pages block_table[b][*]
  const int32_t *seq_lens;  // [B]
  const int32_t *block_table;  // [B][max_pages]
  int max_pages, page_tokens, append, units, B, UH;
  unsigned long long wait_ns;  // bound of every copy wait (WAIT_LIMIT_NS unless a test set one)
  int drop_copies;             // test hook: the scorer issues no copy (its waits run out)
  float *state;                // nullable [B][Hq][D + 2]: the merged state instead of out
};

// Bulk-tensor maps of one decode call.  Values always go through `value`
// (3-D, [B*Hkv][T][d], 128-byte swizzle).  When the context length keeps
// every unit's codes and norms 16-byte aligned (T % 8 == 0), `sign` and
// `norm` map them as [B*Hkv][T*words] and [B*Hkv][T] and one lane fetches a
// whole block; otherwise every lane copies a slice with cp.async.
struct DecMaps {
  CUtensorMap value;
  CUtensorMap sign;
  CUtensorMap norm;
  int tma_codes;  // 1: codes and norms by bulk-tensor copy
  int sign_elem;  // bytes per element of the sign map (4 or 8)
};

// Paged cache: blocks of every unit of sequence b, ceil(len / 32) with
// len = seq_lens[b] (+1 when the call appends a key) kept inside [0, max_len];
// a length outside the bound is reported by the combine.
__device__ __forceinline__ int64_t paged_blocks(const int32_t *seq_lens, int b, int append,
                                                int64_t max_len) {
  int64_t len = (int64_t)__ldg(seq_lens + b) + append;
  len = len < 0 ? 0 : (len > max_len ? max_len : len);
  return (len + DEC_KB - 1) / DEC_KB;
}

// warp that owns block b when NB blocks are cut into W contiguous runs
// starting at floor(w * NB / W)
__host__ __device__ __forceinline__ int warp_of_block(int64_t b, int64_t NB,
                                                      int W) {
  return (int)(((b + 1) * (int64_t)W - 1) / NB);
}

// ---------------------------------------------------------------------------
// 1. query projection u = S q (fp32 accumulate), four vectors per CTA.
//
// y[j][i] = sum_c S[i][c] x_j[c] for x_j = X[x0 + j], j < nx <= 4, written to
// dst[j * M + i].  256 threads: warp w takes sketch rows w, w + 8, ... in
// chunks of 8 rows; lane l holds columns [l*CPL, (l+1)*CPL) of a row, so every
// load of a row is one coalesced 128- or 256-byte line.  The 32 partial sums a
// lane has for a chunk (8 rows x 4 vectors) are combined by a butterfly
// reduce-scatter: 31 shuffles leave lane l with the complete sum of entry l.
constexpr int PROJ_THREADS = 256;
constexpr int PROJ_VECS = 4;

// Extents for the index checks of the debug build: X holds x_extent
// elements, dst (from its start) dst_extent; err null = no checks.
struct ProjLimits {
  int *err = nullptr;
  int64_t x_extent = 0, dst_extent = 0;
};

// RS > 1 splits the m sketch rows over RS CTAs: this CTA projects rows
// [split * m / RS, (split + 1) * m / RS) only (a launch of RS times as many,
// shorter CTAs; the routine is latency-bound, so the split cuts its time).
template <int M, int D, bool XF32, int RS = 1>
__device__ __forceinline__ void project4(const uint16_t *__restrict__ S,
                                         const void *__restrict__ X, int64_t x0,
                                         int nx, float *dst, int dst_stride = M,
                                         const ProjLimits lim = ProjLimits{}, int split = 0) {
  constexpr int CPL = D / 32;        // columns per lane
  constexpr int CH = 8;              // rows per chunk
  constexpr int RPW = M / (8 * RS);  // rows per warp
  static_assert(CH * PROJ_VECS == 32 && RPW % CH == 0 && RPW >= CH, "projection tiling");
  const int rbase = split * (M / RS);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float x[PROJ_VECS][CPL];
#pragma unroll
  for (int j = 0; j < PROJ_VECS; ++j)
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int64_t e = (x0 + j) * D + lane * CPL + c;
      bool ok = j < nx;
      if (ok && lim.err) ok = JL_IN_RANGE(lim.err, e, 1, lim.x_extent);
      x[j][c] = !ok  ? 0.f
                : XF32 ? reinterpret_cast<const float *>(X)[e]
                       : bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(X)[e]);
    }
#pragma unroll
  for (int r0 = 0; r0 < RPW; r0 += CH) {
    uint32_t sw[CH][CPL / 2];
#pragma unroll
    for (int k = 0; k < CH; ++k) {
      const uint16_t *row = S + (int64_t)(rbase + warp + 8 * (r0 + k)) * D + lane * CPL;
      if constexpr (CPL == 4) {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(row));
        sw[k][0] = t.x;
        sw[k][1] = t.y;
      } else {
        sw[k][0] = __ldg(reinterpret_cast<const uint32_t *>(row));
      }
    }
    float v[32];
#pragma unroll
    for (int k = 0; k < CH; ++k)
#pragma unroll
      for (int j = 0; j < PROJ_VECS; ++j) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < CPL / 2; ++c) {
          a = fmaf(__uint_as_float(sw[k][c] << 16), x[j][2 * c], a);
          a = fmaf(__uint_as_float(sw[k][c] & 0xFFFF0000u), x[j][2 * c + 1], a);
        }
        v[k * PROJ_VECS + j] = a;
      }
#pragma unroll
    for (int st = 16; st >= 1; st >>= 1) {
      const bool upper = (lane & st) != 0;
#pragma unroll
      for (int k = 0; k < st; ++k) {
        const float send = upper ? v[k] : v[k + st];
        const float keep = upper ? v[k + st] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, st);
      }
    }
    const int k = lane / PROJ_VECS, j = lane % PROJ_VECS;
    const int64_t di = (int64_t)j * dst_stride + rbase + warp + 8 * (r0 + k);
    if (j < nx && (!lim.err || JL_IN_RANGE(lim.err, di, 1, lim.dst_extent))) dst[di] = v[0];
  }
}

// Row splits of the query projection: one 8-row chunk per warp.
template <int M>
constexpr int proj_splits() {
  return M / 64;
}

template <int M, int D, bool QF32>
__global__ void __launch_bounds__(PROJ_THREADS) qproj_kernel(const void *__restrict__ Q,
                                                             const uint16_t *__restrict__ S,
                                                             float *__restrict__ U, int nq,
                                                             int *err) {
  griddep_launch_dependents();  // let the scorer start its copies now
  const int64_t x0 = (int64_t)blockIdx.x * PROJ_VECS;
  const int nx = (int)min((int64_t)PROJ_VECS, (int64_t)nq - x0);
  project4<M, D, QF32, proj_splits<M>()>(S, Q, x0, nx, U + x0 * M, M,
                                         ProjLimits{err, (int64_t)nq * D, ((int64_t)nq - x0) * M},
                                         (int)blockIdx.y);
}

// TurboQuant-prod query rows, four queries per CTA: w = Pinv^T q (so that
// <w, Pi x> = <q, x> for the stored bf16 Pi), then the row
//   [wc_0 w, ..., wc_{TERMS-1} w, 0..., S w, 0...]
// (each segment zero-padded to whole 128-coordinate runs, TurboRow)
// whose dot product with the +-1 expansion of a key's code [plane terms,
// signs] gives the two raw sums of the score: the plane terms' part is
// <w, c[cell]> because a symmetric codebook is the sum of its odd Walsh
// terms, c_j = sum_S wc_S prod_{p in S} (2 bit_p(j) - 1) over the odd subsets
// S of the planes (the single planes, and for three planes also all three).
struct WalshCoef {
  float c[4];  // coefficients of the plane terms, in code order
};

template <int M, int D, int TB, bool QF32>
__device__ __forceinline__ void turbo_query_rows(const void *__restrict__ Q,
                                                 const float *__restrict__ Pinv,
                                                 const uint16_t *__restrict__ S,
                                                 float *__restrict__ U, int nq,
                                                 const WalshCoef &wc, int64_t x0,
                                                 int *err) {
  using R = TurboRow<M, D, TB>;
  constexpr int TERMS = R::TERMS;
  constexpr int MT = R::LEN;
  constexpr int HALVES = PROJ_THREADS / D;  // threads per output coordinate
  static_assert(PROJ_THREADS % D == 0 && D % HALVES == 0, "query map tiling");
  __shared__ float qsm[PROJ_VECS * D];
  __shared__ float part[HALVES][PROJ_VECS * D];
  __shared__ float wsm[PROJ_VECS * D];
  const int nx = (int)min((int64_t)PROJ_VECS, (int64_t)nq - x0);
  for (int e = threadIdx.x; e < PROJ_VECS * D; e += PROJ_THREADS) {
    const int j = e / D;
    const int64_t src = x0 * D + e;
    qsm[e] = (j >= nx || !JL_IN_RANGE(err, src, 1, (int64_t)nq * D)) ? 0.f
             : QF32 ? reinterpret_cast<const float *>(Q)[src]
                    : bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(Q)[src]);
  }
  __syncthreads();
  {
    // thread (i, h): partial sums over columns c of part h, all four queries
    // at once so that each Pinv element is read once
    const int i = threadIdx.x % D, h = threadIdx.x / D;
    constexpr int CP = D / HALVES;
    float acc[PROJ_VECS] = {};
    // all of the thread's Pinv loads in flight at once (one L2 round trip,
    // not one per group of eight)
    float pv[CP];
#pragma unroll
    for (int cc = 0; cc < CP; ++cc) pv[cc] = __ldg(Pinv + (h * CP + cc) * D + i);
#pragma unroll
    for (int cc = 0; cc < CP; ++cc)
#pragma unroll
      for (int j = 0; j < PROJ_VECS; ++j)
        acc[j] = fmaf(pv[cc], qsm[j * D + h * CP + cc], acc[j]);
#pragma unroll
    for (int j = 0; j < PROJ_VECS; ++j) part[h][j * D + i] = acc[j];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < PROJ_VECS * D; e += PROJ_THREADS) {
    float w = 0.f;
#pragma unroll
    for (int h = 0; h < HALVES; ++h) w += part[h][e];
    wsm[e] = w;
  }
  __syncthreads();
  project4<M, D, true>(S, wsm, 0, nx, U + x0 * MT + R::MSE, MT,
                       ProjLimits{err, PROJ_VECS * D, ((int64_t)nq - x0) * MT - R::MSE});
  for (int e = threadIdx.x; e < nx * D; e += PROJ_THREADS) {
    const int j = e / D, i = e - (e / D) * D;
    float *row = U + (x0 + j) * MT;
#pragma unroll
    for (int k = 0; k < TERMS; ++k)
      if (JL_IN_RANGE(err, (x0 + j) * MT + k * D + i, 1, (int64_t)nq * MT))
        row[k * D + i] = wc.c[k] * wsm[e];
  }
  if constexpr (R::MSE > TERMS * D || R::QJL > M) {
    // the padding of both segments
    constexpr int P1 = R::MSE - TERMS * D, P2 = R::QJL - M;
    for (int e = threadIdx.x; e < nx * (P1 + P2); e += PROJ_THREADS) {
      const int j = e / (P1 + P2), c = e - j * (P1 + P2);
      const int col = c < P1 ? TERMS * D + c : R::MSE + M + (c - P1);
      if (JL_IN_RANGE(err, (x0 + j) * MT + col, 1, (int64_t)nq * MT)) U[(x0 + j) * MT + col] = 0.f;
    }
  }
}

template <int M, int D, int TB, bool QF32>
__global__ void __launch_bounds__(PROJ_THREADS)
    turbo_qproj_kernel(const void *__restrict__ Q, const float *__restrict__ Pinv,
                       const uint16_t *__restrict__ S, float *__restrict__ U, int nq,
                       const WalshCoef wc, int *err) {
  griddep_launch_dependents();
  turbo_query_rows<M, D, TB, QF32>(Q, Pinv, S, U, nq, wc, (int64_t)blockIdx.x * PROJ_VECS,
                                   err);
}

// ---------------------------------------------------------------------------
// 2. scorer

// Position of a block in the (unit, block) space, advanced without division,
// with the geometry of its unit: blocks nb, keys len, kv row kvi = b*Hkv + hkv.
struct BlockPos {
  int64_t u;    // unit
  int64_t blk;  // block within the unit
  int64_t nb;   // blocks of unit u
  int64_t len;  // keys of unit u
  int64_t kvi;  // b * Hkv + kv head of unit u
  // paged cache only: the block's page within its sequence (pidx), its first
  // row in that page (y), the sequence's block-table row, the kv head, and
  // the pool page itself once looked up (load_page); kept up to date without
  // divisions as the position advances
  int pidx, y, hkv, page;
  const int32_t *trow;
};

template <bool PAGED>
__device__ __forceinline__ void pos_load_unit(const DecParams &p, BlockPos &pos) {
  pos.kvi = p.HG == 1 ? pos.u : pos.u / p.HG;
  if constexpr (PAGED) {
    const int b = (int)pos.kvi / p.Hkv;  // kv rows < 2^24 (checked by the plan)
    pos.hkv = (int)pos.kvi - b * p.Hkv;
    pos.trow = p.block_table + (int64_t)b * p.max_pages;
    pos.nb = paged_blocks(p.seq_lens, b, p.append, p.T);
    // keep every access inside the bound, whatever the length says
    const int64_t len = (int64_t)__ldg(p.seq_lens + b) + p.append;
    pos.len = len < 0 ? 0 : (len < p.T ? len : p.T);
  } else {
    pos.nb = p.nb_u;
    pos.len = p.T;
  }
}

// Position of flat block b (which must exist), contiguous cache.
__device__ __forceinline__ BlockPos pos_of_block(const DecParams &p, int64_t b) {
  BlockPos pos;
  pos.u = b / p.nb_u;
  pos.blk = b - pos.u * p.nb_u;
  pos_load_unit<false>(p, pos);
  return pos;
}

// Paged cache, whole warp: total blocks NB of the flat space (sum over the
// sequences of UH * paged_blocks), the same in every lane.  Not inlined: it
// runs once per warp and keeps its registers out of the streaming loop.
__device__ __noinline__ int64_t paged_total(const int32_t *seq_lens, int B, int append,
                                            int64_t max_len, int UH, int lane) {
  int64_t tot = 0;
  for (int b = lane; b < B; b += 32) tot += paged_blocks(seq_lens, b, append, max_len);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  return tot * UH;
}

// Paged cache, whole warp: the sequence whose range of the flat block space
// holds block bb (b = -1 if none does), with the range's first block and the
// blocks of each of its units.  A scan over the sequences, 32 at a time.
struct SeqHit {
  int64_t start, nbs;
  int b;
};
__device__ __noinline__ SeqHit paged_find(const int32_t *seq_lens, int B, int append,
                                          int64_t max_len, int UH, int64_t bb, int lane) {
  int64_t carry = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const int64_t n = b < B ? paged_blocks(seq_lens, b, append, max_len) * UH : 0;
    int64_t incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int64_t excl = carry + incl - n;
    const uint32_t hit = __ballot_sync(0xffffffffu, n > 0 && excl <= bb && bb < excl + n);
    if (hit) {
      const int src = __ffs(hit) - 1;
      SeqHit h;
      h.start = __shfl_sync(0xffffffffu, excl, src);
      h.nbs = __shfl_sync(0xffffffffu, n, src) / UH;
      h.b = b0 + src;
      return h;
    }
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  SeqHit none;
  none.start = none.nbs = 0;
  none.b = -1;
  return none;
}

// TRACK: keep the page fields up to date (positions that issue copies).
template <bool PAGED, bool TRACK = true>
__device__ __forceinline__ void pos_next(const DecParams &p, BlockPos &pos) {
  if (++pos.blk < pos.nb) {
    if constexpr (PAGED && TRACK) {
      pos.y += DEC_KB;  // pages hold a whole number of blocks
      if (pos.y == p.page_tokens) {
        pos.y = 0;
        ++pos.pidx;
      }
    }
    return;
  }
  pos.blk = 0;
  if constexpr (PAGED) {
    if constexpr (TRACK) {
      pos.y = 0;
      pos.pidx = 0;
    }
    // skip units without blocks; never step past the last unit
    do {
      if (pos.u + 1 >= p.units) return;
      ++pos.u;
      pos_load_unit<PAGED>(p, pos);
    } while (pos.nb == 0);
  } else {
    ++pos.u;
    pos_load_unit<PAGED>(p, pos);
  }
}

// Paged cache: look up the pool page of the block at `pos` ahead of the copy
// that needs it, so that the table read is not on the issue path.  `pos` is
// always a block of its unit or block 0 of a unit, so the entry read lies
// inside the sequence's row of the table.
__device__ __forceinline__ void load_page(BlockPos &pos) {
  pos.page = __ldg(pos.trow + pos.pidx);
}

template <int M, int D, bool S8, int TB = 0>
struct Ring {
  using C = DecCfg<M, D, S8, TB>;
  uint32_t base;   // this warp's stages (1024-aligned)
  uint32_t nbase;  // this warp's norm areas
  uint32_t bbase;  // this warp's barriers
  __device__ __forceinline__ uint32_t val(int s) const { return base + s * C::STAGE_BYTES; }
  __device__ __forceinline__ uint32_t sign(int s) const {
    return base + s * C::STAGE_BYTES + C::V_BYTES;
  }
  __device__ __forceinline__ uint32_t afrag() const { return base + C::STAGES * C::STAGE_BYTES; }
  __device__ __forceinline__ uint32_t norm(int s) const { return nbase + s * C::NORM_AREA; }
  __device__ __forceinline__ uint32_t bar(int s) const { return bbase + 8 * s; }
};

// Start the copies of block `pos` into stage s: values by one 3-D bulk-tensor
// copy per 64 columns (lane 0), codes and norms by cp.async (all lanes).
template <int M, int D, bool S8, bool PAGED, int TB = 0>
__device__ __forceinline__ void issue_block(const DecParams &p, const DecMaps &maps,
                                            const Ring<M, D, S8, TB> &ring, const BlockPos &pos,
                                            int s, int lane) {
  using C = DecCfg<M, D, S8, TB>;
  if (p.drop_copies) return;
  const int64_t kvi = pos.kvi;
  const int64_t key0 = pos.blk * DEC_KB;
  if (PAGED || maps.tma_codes) {
    if (lane == 0) {
      // row (y) within the tensor's unit (z): the sequence itself, or the page
      // holding this block (row within the page) for a paged cache
      int y = (int)key0, z = (int)kvi;
      if constexpr (PAGED) {
        y = pos.y;
        z = pos.page * p.Hkv + pos.hkv;
      }
      mbar_expect_tx(ring.bar(s), C::V_BYTES + C::SIGN_BYTES + C::NORM_BYTES * DEC_KB);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(ring.val(s) + h * C::V_BOX, &maps.value, h * 64, y, z, ring.bar(s));
      tma_load_2d(ring.sign(s), &maps.sign, (int)((int64_t)y * C::KEY_SIGN_BYTES / maps.sign_elem),
                  z, ring.bar(s));
      tma_load_2d(ring.norm(s), &maps.norm, y, z, ring.bar(s));
    }
    return;
  }
  const int64_t left = p.T - key0;
  const int nval = left < DEC_KB ? (int)left : DEC_KB;
  const int64_t gkey = kvi * p.T + key0;
  // codes: SIGN_BYTES contiguous bytes, a slice per lane, zero past the context
  const uint8_t *sg = reinterpret_cast<const uint8_t *>(p.signs) + gkey * C::KEY_SIGN_BYTES;
  const uint32_t sdst = ring.sign(s);
#pragma unroll
  for (int e = lane; e < C::SIGN_CHUNKS; e += 32) {
    const bool ok = e * C::SIGN_CHUNK < nval * C::KEY_SIGN_BYTES &&
                    JL_IN_RANGE(p.err, gkey * C::KEY_SIGN_BYTES + e * C::SIGN_CHUNK,
                                C::SIGN_CHUNK, p.n_keys * C::KEY_SIGN_BYTES);
    const void *src = ok ? (const void *)(sg + e * C::SIGN_CHUNK) : (const void *)p.signs;
    if constexpr (C::SIGN_CHUNK == 16)
      cp_async_16(sdst + e * 16, src, ok ? 16 : 0);
    else
      cp_async_8(sdst + e * 8, src, ok ? 8 : 0);
  }
  // norms: the 16-byte-aligned run of G-key groups covering the block (G = 8
  // binary16 norms, or 4 pairs); key k of the block lands at key slot
  // (gkey % G) + k
  constexpr int G = 16 / C::NORM_BYTES;
  constexpr int GROUPS = (DEC_KB + G - 1) / G + 1;
  if (lane < GROUPS) {
    const int64_t first = (gkey & ~(int64_t)(G - 1)) + G * lane;
    const int64_t avail = p.n_keys - first;
    bool ok = first < gkey + nval && avail > 0;
    const int nbytes0 = ok ? (avail >= G ? 16 : (int)avail * C::NORM_BYTES) : 0;
    if (ok) ok = JL_IN_RANGE(p.err, first * C::NORM_BYTES, nbytes0, p.n_keys * C::NORM_BYTES);
    const int nbytes = ok ? nbytes0 : 0;
    const uint8_t *nb = reinterpret_cast<const uint8_t *>(p.norms);
    cp_async_16(ring.norm(s) + 16 * lane,
                ok ? (const void *)(nb + first * C::NORM_BYTES) : (const void *)nb, nbytes);
  }
  cp_async_mbar_arrive(ring.bar(s));
  __syncwarp();
  if (lane == 0) {
    mbar_expect_tx(ring.bar(s), C::V_BYTES);
#pragma unroll
    for (int h = 0; h < D / 64; ++h)
      tma_load_3d(ring.val(s) + h * C::V_BOX, &maps.value, h * 64, (int)key0, (int)kvi,
                  ring.bar(s));
  }
}


__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// The lane's 32-coordinate runs of u: lane t of a quad owns code words
// t*M/128 .. (M >= 128), or half of word t/2 (M = 64).  run(k) gives the
// start of the k-th run of `len` consecutive coordinates.
template <int M>
struct LaneRuns {
  static constexpr int WORDS = (M >= 128) ? M / 128 : 1;
};

__device__ __forceinline__ float4 ldg4(const float *p) {
  return __ldg(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ float f4c(const float4 &v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// A fragments of one unit for the lane (g, t): rows 0..7 of the scoring MMA
// hold the high part of S q of the <= 8 heads, rows 8..15 the low part.
//   bf16: hi = bf16(u), lo = bf16(u - hi)
//   int8: u ~= hscale * (256 hi + lo), |256 hi + lo| <= 32000, usum = sum of
//         256 hi + lo over the head's coordinates.
// u is read as whole 16-byte vectors of the lane's own coordinate runs.
template <int M, int D, bool S8, int TB = 0>
__device__ __forceinline__ void build_afrags(const float *urow, bool live, int t,
                                             const Ring<M, D, S8, TB> &ring,
                                             uint32_t (&afr)[DecCfg<M, D, S8, TB>::A_SMEM ? 1 : DecCfg<M, D, S8, TB>::NC][4],
                                             float (&hscale)[2], int (&usum)[2]) {
  using C = DecCfg<M, D, S8, TB>;
  auto put = [&](int c, const uint32_t (&a4)[4]) {
    if constexpr (C::A_SMEM) {
      const int lane = (threadIdx.x & 31);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                       ring.afrag() + (c * 32 + lane) * 16),
                   "r"(a4[0]), "r"(a4[1]), "r"(a4[2]), "r"(a4[3])
                   : "memory");
    } else {
      afr[c][0] = a4[0]; afr[c][1] = a4[1]; afr[c][2] = a4[2]; afr[c][3] = a4[3];
    }
  };
  if constexpr (!S8) {
    if constexpr (C::CODE_BITS >= 128) {
#pragma unroll
      for (int lw = 0; lw < C::LW; ++lw) {
        // code word of the lane's run lw: contiguous runs, or (cell planes)
        // interleaved so that run lw of the four lanes is one plane
        const int word = TB ? 4 * lw + t : t * C::LW + lw;
        const float *src = urow + 32 * word;
        float4 x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = live ? ldg4(src + 4 * k) : make_float4(0, 0, 0, 0);
        // pair p of the word: coordinates p and p + 16 -> chunk 8 lw + p/2, slot p&1
#pragma unroll
        for (int c2 = 0; c2 < 8; ++c2) {
          uint32_t a4[4];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int pp = 2 * c2 + r;
            const float x0 = f4c(x[pp >> 2], pp & 3), x1 = f4c(x[(pp + 16) >> 2], pp & 3);
            const float h0 = bf16_round_f32(x0), h1 = bf16_round_f32(x1);
            a4[2 * r] = pack_bf16x2(h0, h1);
            a4[2 * r + 1] = pack_bf16x2(x0 - h0, x1 - h1);
          }
          put(8 * lw + c2, a4);
        }
      }
    } else {
      // M = 64: pairs 8(t&1) .. +7 of word t/2
      const float *src = urow + 32 * (t >> 1) + 8 * (t & 1);
      float4 x[4];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        x[k] = live ? ldg4(src + 4 * k) : make_float4(0, 0, 0, 0);
        x[2 + k] = live ? ldg4(src + 16 + 4 * k) : make_float4(0, 0, 0, 0);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t a4[4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int q = 2 * c + r;
          const float x0 = f4c(x[q >> 2], q & 3), x1 = f4c(x[2 + (q >> 2)], q & 3);
          const float h0 = bf16_round_f32(x0), h1 = bf16_round_f32(x1);
          a4[2 * r] = pack_bf16x2(h0, h1);
          a4[2 * r + 1] = pack_bf16x2(x0 - h0, x1 - h1);
        }
        put(c, a4);
      }
    }
    (void)hscale; (void)usum;
  } else if constexpr (TB > 0) {
    // cell-plane codes: lane t owns code words 4 lw + t; runs lw < TB are
    // cell planes (the codebook-weighted w), the others residual signs (S w):
    // one scale per segment, u ~= hscale[s] (256 hi + lo), |256 hi + lo| <= 32000
    float am[2] = {0.f, 0.f};
    if (live) {
#pragma unroll
      for (int lw = 0; lw < C::LW; ++lw) {
        const float *src = urow + 32 * (4 * lw + t);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 v = ldg4(src + 4 * k);
          const float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
          am[lw < C::MSE_RUNS ? 0 : 1] = fmaxf(am[lw < C::MSE_RUNS ? 0 : 1], a);
        }
      }
    }
    float inv[2];
#pragma unroll
    for (int sg = 0; sg < 2; ++sg) {
      am[sg] = fmaxf(am[sg], __shfl_xor_sync(0xffffffffu, am[sg], 1));
      am[sg] = fmaxf(am[sg], __shfl_xor_sync(0xffffffffu, am[sg], 2));
      hscale[sg] = am[sg] > 0.f ? am[sg] / 32000.f : 0.f;
      inv[sg] = am[sg] > 0.f ? 32000.f / am[sg] : 0.f;
    }
    int isum[2] = {0, 0};
#pragma unroll
    for (int lw = 0; lw < C::LW; ++lw) {
      const int sg = lw < C::MSE_RUNS ? 0 : 1;
      const float *src = urow + 32 * (4 * lw + t);
      float4 x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = live ? ldg4(src + 4 * k) : make_float4(0, 0, 0, 0);
      // byte register p of the word holds coordinates p + 8j, j = 0..3
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        uint32_t a4[4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int pp = 2 * c2 + r;
          int hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int ui = __float2int_rn(f4c(x[(pp + 8 * j) >> 2], pp & 3) * inv[sg]);
            isum[sg] += ui;
            hi[j] = (ui + 128) >> 8;
            lo[j] = ui - (hi[j] << 8);
          }
          a4[2 * r] = pack_s8x4(hi[0], hi[1], hi[2], hi[3]);
          a4[2 * r + 1] = pack_s8x4(lo[0], lo[1], lo[2], lo[3]);
        }
        put(4 * lw + c2, a4);
      }
    }
#pragma unroll
    for (int sg = 0; sg < 2; ++sg) {
      isum[sg] += __shfl_xor_sync(0xffffffffu, isum[sg], 1);
      isum[sg] += __shfl_xor_sync(0xffffffffu, isum[sg], 2);
      usum[sg] = isum[sg];
    }
  } else {
    // pass 1: the head's largest |u| (4 lanes of the quad together)
    float amax = 0.f;
    if (live) {
      if constexpr (M >= 128) {
#pragma unroll
        for (int lw = 0; lw < LaneRuns<M>::WORDS; ++lw) {
          const float *src = urow + 32 * (t * LaneRuns<M>::WORDS + lw);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 v = ldg4(src + 4 * k);
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
          }
        }
      } else {
        const float *src = urow + 32 * (t >> 1) + 4 * (t & 1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 v = ldg4(src + 8 * j);
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
      }
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    hscale[0] = amax > 0.f ? amax / 32000.f : 0.f;
    const float inv = amax > 0.f ? 32000.f / amax : 0.f;
    int isum = 0;
    auto quant = [&](float x, int &hi, int &lo) {
      const int ui = __float2int_rn(x * inv);
      isum += ui;
      hi = (ui + 128) >> 8;
      lo = ui - (hi << 8);
    };
    // pass 2: byte register p of a word holds coordinates p + 8j, j = 0..3
    if constexpr (M >= 128) {
#pragma unroll
      for (int lw = 0; lw < LaneRuns<M>::WORDS; ++lw) {
        const float *src = urow + 32 * (t * LaneRuns<M>::WORDS + lw);
        float4 x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = live ? ldg4(src + 4 * k) : make_float4(0, 0, 0, 0);
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          uint32_t a4[4];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int pp = 2 * c2 + r;
            int hi[4], lo[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) quant(f4c(x[(pp + 8 * j) >> 2], pp & 3), hi[j], lo[j]);
            a4[2 * r] = pack_s8x4(hi[0], hi[1], hi[2], hi[3]);
            a4[2 * r + 1] = pack_s8x4(lo[0], lo[1], lo[2], lo[3]);
          }
          put(4 * lw + c2, a4);
        }
      }
    } else {
      const float *src = urow + 32 * (t >> 1) + 4 * (t & 1);
      float4 x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = live ? ldg4(src + 8 * j) : make_float4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t a4[4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int q = 2 * c + r;
          int hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) quant(f4c(x[j], q), hi[j], lo[j]);
          a4[2 * r] = pack_s8x4(hi[0], hi[1], hi[2], hi[3]);
          a4[2 * r + 1] = pack_s8x4(lo[0], lo[1], lo[2], lo[3]);
        }
        put(c, a4);
      }
    }
    isum += __shfl_xor_sync(0xffffffffu, isum, 1);
    isum += __shfl_xor_sync(0xffffffffu, isum, 2);
    usum[0] = isum;
  }
  if constexpr (C::A_SMEM) __syncwarp();
}

// Query fragments of the int8 scoring with the keys as the MMA's rows (at
// most four query heads per KV head): the B operand of m16n8k32 holds head
// h's quantised u in columns 2h (high limbs) and 2h + 1 (low limbs), columns
// of absent heads zero.  u is quantised exactly as build_afrags does it (per
// head to +-32000, two limbs, the same coordinate order: k slot 4t + i of
// slice c is bit (2c & 7) + 8i of the lane's word t * WORDS + c / 4, and slot
// 16 + 4t + i bit (2c & 7) + 1 + 8i), so column g of lane (g, t) needs the
// limbs of head g / 2: lanes 2h and 2h + 1 both quantise head h's row (urow,
// live) and keep one limb each; hscale / usum come back per lane group.
template <int M, int D, int TB = 0>
__device__ __forceinline__ void build_bfrags_keyrows(const float *urow, bool live, int g, int t,
                                                     uint32_t (&bfr)[DecCfg<M, D, true, TB>::NC][2],
                                                     float (&hscale)[2], int (&usum)[2]) {
  using C = DecCfg<M, D, true, TB>;
  static_assert(TB > 0 || M >= 128, "keys-as-rows scoring: m >= 128");
  // runs of 32-coordinate words the lane reads: contiguous (QJL codes) or,
  // for cell-plane codes, word 4 lw + t with segment (planes, residual signs)
  // by run, as build_afrags
  constexpr int RUNS = TB ? C::LW : LaneRuns<M>::WORDS;
  auto word_of = [&](int lw) { return TB ? 4 * lw + t : t * RUNS + lw; };
  auto seg_of = [&](int lw) { return (TB && lw >= C::MSE_RUNS) ? 1 : 0; };
  float am[2] = {0.f, 0.f};
  if (live) {
#pragma unroll
    for (int lw = 0; lw < RUNS; ++lw) {
      const float *src = urow + 32 * word_of(lw);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 v = ldg4(src + 4 * k);
        am[seg_of(lw)] = fmaxf(am[seg_of(lw)],
                               fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
  }
  float inv[2];
#pragma unroll
  for (int sg = 0; sg < 2; ++sg) {
    am[sg] = fmaxf(am[sg], __shfl_xor_sync(0xffffffffu, am[sg], 1));
    am[sg] = fmaxf(am[sg], __shfl_xor_sync(0xffffffffu, am[sg], 2));
    hscale[sg] = am[sg] > 0.f ? am[sg] / 32000.f : 0.f;
    inv[sg] = am[sg] > 0.f ? 32000.f / am[sg] : 0.f;
  }
  int isum[2] = {0, 0};
#pragma unroll
  for (int lw = 0; lw < RUNS; ++lw) {
    const int sg = seg_of(lw);
    const float *src = urow + 32 * word_of(lw);
    float4 x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = live ? ldg4(src + 4 * k) : make_float4(0, 0, 0, 0);
#pragma unroll
    for (int c2 = 0; c2 < 4; ++c2) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int pp = 2 * c2 + r;
        int hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ui = __float2int_rn(f4c(x[(pp + 8 * j) >> 2], pp & 3) * inv[sg]);
          isum[sg] += ui;
          hi[j] = (ui + 128) >> 8;
          lo[j] = ui - (hi[j] << 8);
        }
        // column g: head g / 2, the high (g even) or low (g odd) limb
        bfr[4 * lw + c2][r] = !live        ? 0u
                              : (g & 1) == 0 ? pack_s8x4(hi[0], hi[1], hi[2], hi[3])
                                             : pack_s8x4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
  }
#pragma unroll
  for (int sg = 0; sg < 2; ++sg) {
    isum[sg] += __shfl_xor_sync(0xffffffffu, isum[sg], 1);
    isum[sg] += __shfl_xor_sync(0xffffffffu, isum[sg], 2);
    usum[sg] = isum[sg];
  }
}

// KR: int8 scoring with the keys as the MMA's rows (at most four query heads
// per KV head, m >= 128, QJL codes): 16 keys per m16n8k32, the eight columns
// the two limbs of each head; half the MMAs of the head-rows form, whose
// 16 rows then hold at most eight live limb rows.
template <int M, int D, bool S8, bool PAGED, int TB = 0, bool KR = false>
__global__ void __launch_bounds__(DEC_WARPS * 32)
    decode_scorer_kernel(const __grid_constant__ DecMaps maps, const DecParams p) {
  using C = DecCfg<M, D, S8, TB>;
  static_assert(!KR || (S8 && (TB > 0 || M >= 128)), "keys-as-rows scoring: int8, m >= 128");
  // (a keys-as-rows launch has at most four heads per unit: p.G <= 4)
  extern __shared__ uint8_t dsmem_raw[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int w = blockIdx.x * DEC_WARPS + wid;
  if (w >= p.W) return;
  // a paged call plans its split from seq_lens (an input, not written by the
  // prep kernel that runs before this one); it is launched for the bound, so
  // with fewer blocks than warps the first NB warps take one block each and
  // the rest have nothing to do (no warp may own an empty run: the combine
  // reads a record from every warp between a unit's first and last)
  const int64_t NB =
      PAGED ? paged_total(p.seq_lens, p.B, p.append, p.T, p.UH, lane) : p.NB;
  const int Wn = PAGED ? (int)(NB < p.W ? NB : p.W) : p.W;
  if (w >= Wn) return;
  const int g = lane >> 2;  // group id: head row / key column / dim row
  const int t = lane & 3;   // thread in group
  const uint32_t cta = (smem_u32(dsmem_raw) + 1023u) & ~1023u;
  const Ring<M, D, S8, TB> ring{cta + wid * C::WARP_BYTES,
                        cta + C::OFF_NORM + wid * C::STAGES * C::NORM_AREA,
                        cta + C::OFF_BAR + wid * C::STAGES * 8};

  const int64_t bbeg = (int64_t)w * NB / Wn;
  const int64_t bend = (int64_t)(w + 1) * NB / Wn;
  const int64_t nblk = bend - bbeg;
  if (nblk <= 0) return;

  if (lane == 0)
    for (int s = 0; s < C::STAGES; ++s) mbar_init(ring.bar(s), 1);
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  __syncwarp();

  // prologue: fill the ring
  BlockPos ipos;
  if constexpr (PAGED) {
    const SeqHit h = paged_find(p.seq_lens, p.B, p.append, p.T, p.UH, bbeg, lane);
    if (h.b < 0) {
      if (lane == 0) record_device_error(p.err, DERR_DECODE_PLAN);
      return;
    }
    const int64_t r = bbeg - h.start;
    const int64_t uin = r / h.nbs;
    ipos.u = (int64_t)h.b * p.UH + uin;
    ipos.blk = r - uin * h.nbs;
    pos_load_unit<true>(p, ipos);
    const int key0 = (int)ipos.blk * DEC_KB;  // < max_len < 2^31
    ipos.pidx = key0 / p.page_tokens;
    ipos.y = key0 - ipos.pidx * p.page_tokens;
    load_page(ipos);
  } else {
    ipos = pos_of_block(p, bbeg);
  }
  const BlockPos pos0 = ipos;
  int issued = 0;
#pragma unroll
  for (int s = 0; s < C::STAGES; ++s) {
    if (s < nblk) {
      // the block holding the key this call appends is written by the prep
      // kernel: copy it only after the wait below
      if (PAGED && p.append && ipos.blk == ipos.nb - 1) break;
      issue_block<M, D, S8, PAGED, TB>(p, maps, ring, ipos, s, lane);
      pos_next<PAGED>(p, ipos);
      if constexpr (PAGED) load_page(ipos);
      ++issued;
    }
  }

  // the query projections (and a paged call's appended keys) come from the
  // previous kernel on the stream, which may still be running (programmatic
  // dependent launch): wait for it only now, after the first copies are on
  // their way
  griddep_wait();
  for (int s = issued; s < C::STAGES && s < nblk; ++s) {
    issue_block<M, D, S8, PAGED, TB>(p, maps, ring, ipos, s, lane);
    pos_next<PAGED>(p, ipos);
    if constexpr (PAGED) load_page(ipos);
  }

  // per-unit state
  int64_t cur_u = -1, kv_base = 0;
  int Gg = 0, b_idx = 0, hq0 = 0;
  float mx = -INFINITY, lsum = 0.f;
  // int8 scoring: value of one unit of the query row for head g and the sum
  // of its quantized entries, per segment (cell planes, residual signs)
  float hscale[2] = {0.f, 0.f};
  int usum[2] = {0, 0};
  float acc[C::DT][4];
  uint32_t afr[(C::A_SMEM || KR) ? 1 : C::NC][4];
  uint32_t bfr[KR ? C::NC : 1][2];
  // a wait that ran out: bit 0 = it did; bits 1-2 = the block's index mod 4
  // (its stage and phase); bit 3 = the next block was started too
  int failed = 0;

  auto flush = [&](int64_t u) {
    float l = lsum;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    // the warps of unit u are warp_of_block(first block of u) .. ; warp w's
    // record for unit u is w + u: a warp's records are consecutive, and the
    // next warp's first record comes after its last
    const int64_t rec_idx = (int64_t)w + u;
    if (rec_idx >= p.slots) {
      record_device_error(p.err, DERR_DECODE_PLAN);
      return;
    }
    float *rec = p.partials + (size_t)rec_idx * DEC_HPAD * (D + 2);
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
    const int64_t left = pos.len - key0;
    const int nval = left < DEC_KB ? (int)left : DEC_KB;

    if (u != cur_u) {
      if (cur_u >= 0) flush(cur_u);
      cur_u = u;
      const int kvi = (int)pos.kvi;  // < 2^24 (checked by the plan)
      const int hg = (int)u - kvi * p.HG;
      b_idx = kvi / p.Hkv;
      const int hkv = kvi - b_idx * p.Hkv;
      kv_base = (int64_t)kvi * p.T;
      hq0 = hkv * p.G + hg * DEC_HPAD;
      Gg = min(DEC_HPAD, p.G - hg * DEC_HPAD);
      mx = -INFINITY;
      lsum = 0.f;
#pragma unroll
      for (int dt = 0; dt < C::DT; ++dt)
        acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
      const float *urow = p.U + ((int64_t)b_idx * p.Hq + hq0 + g) * C::CODE_BITS;
      const bool live =
          g < Gg && JL_IN_RANGE(p.err, ((int64_t)b_idx * p.Hq + hq0 + g) * C::CODE_BITS,
                                C::CODE_BITS, (int64_t)p.B * p.Hq * C::CODE_BITS);
      if constexpr (KR) {
        // lanes 2h and 2h + 1 quantise head h's row (one limb each); lane
        // (g, t) then takes head g's scale and sum for the softmax layout
        const int hb = g >> 1;
        const float *urowb = p.U + ((int64_t)b_idx * p.Hq + hq0 + hb) * C::CODE_BITS;
        const bool liveb =
            hb < Gg && JL_IN_RANGE(p.err, ((int64_t)b_idx * p.Hq + hq0 + hb) * C::CODE_BITS,
                                   C::CODE_BITS, (int64_t)p.B * p.Hq * C::CODE_BITS);
        build_bfrags_keyrows<M, D, TB>(urowb, liveb, g, t, bfr, hscale, usum);
#pragma unroll
        for (int sg = 0; sg < (TB ? 2 : 1); ++sg) {
          hscale[sg] = __shfl_sync(0xffffffffu, hscale[sg], (8 * g) & 31);
          usum[sg] = __shfl_sync(0xffffffffu, usum[sg], (8 * g) & 31);
        }
        (void)urow;
        (void)live;
      } else {
        build_afrags<M, D, S8, TB>(urow, live, t, ring, afr, hscale, usum);
      }
      if constexpr (C::A_SMEM) __syncwarp();
    }

    // the lanes wait converged, so they read the same barrier state and the
    // same timer at the same instructions and agree on the outcome (the code
    // below is warp-synchronous)
    __syncwarp();
    if (!mbar_wait_bounded(ring.bar(s), (uint32_t)((i / C::STAGES) & 1), p.wait_ns)) {
      record_device_error(p.err, DERR_DECODE_WAIT_TIMEOUT);
      failed = 1 | ((int)(i & 3) << 1) | (i + 1 < nblk ? 8 : 0);
      break;
    }
    if constexpr (PAGED) {
      // a page's slots past the sequence's last key hold whatever was there:
      // zero those value rows so that p = 0 cannot meet a NaN
      if (nval < DEC_KB) {
        const uint32_t vb = ring.val(s);
        for (int e = lane; e < (DEC_KB - nval) * (D / 64) * 8; e += 32) {
          const int row = nval + e / ((D / 64) * 8);
          const int rest = e - (row - nval) * ((D / 64) * 8);
          const uint32_t addr = vb + (rest >> 3) * C::V_BOX + row * 128 + (rest & 7) * 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};\n" ::"r"(addr), "r"(0)
                       : "memory");
        }
        // the stage is refilled by bulk-tensor copies later: order these
        // generic-proxy writes before them
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
      }
    }

    // ---- code words of the 4 groups of 8 keys (lane: key kg*8 + g)
    const uint32_t sg = ring.sign(s);
    uint32_t wd[4][C::LW];
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) {
      const uint32_t kp = sg + (kg * 8 + g) * C::KEY_SIGN_BYTES;
      if constexpr (TB > 0 && D == 64) {
        // run lw, lane t: logical word L = 4 lw + t of the padded row; plane
        // words are stored first (2 per plane), then the residual signs; the
        // product term's word (TB = 3) is the XOR of the three planes'; a
        // padding word is 0 (its query weights are 0)
        constexpr int PW = D / 32;
#pragma unroll
        for (int lw = 0; lw < C::LW; ++lw) {
          const int L = 4 * lw + t;
          uint32_t w = 0u;
          if (lw < C::MSE_RUNS) {
            if (L < TB * PW) {
              asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(w) : "r"(kp + L * 4));
            } else if (TB == 3 && L < C::TERMS * PW) {
              const int x = L - 3 * PW;
              uint32_t w0, w1, w2;
              asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(w0) : "r"(kp + x * 4));
              asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(w1) : "r"(kp + (PW + x) * 4));
              asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(w2) : "r"(kp + (2 * PW + x) * 4));
              w = w0 ^ w1 ^ w2;
            }
          } else {
            const int jw = L - 4 * C::MSE_RUNS;
            if (jw < M / 32)
              asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(w) : "r"(kp + (TB * PW + jw) * 4));
          }
          wd[kg][lw] = w;
        }
      } else if constexpr (TB == 3) {
        // stored words: planes 0-2, then the residual signs; the product
        // term's word is the XOR of the three planes
#pragma unroll
        for (int lw = 0; lw < 3; ++lw)
          asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(wd[kg][lw]) : "r"(kp + (4 * lw + t) * 4));
        asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(wd[kg][4]) : "r"(kp + (12 + t) * 4));
        wd[kg][3] = wd[kg][0] ^ wd[kg][1] ^ wd[kg][2];
      } else if constexpr (TB > 0) {
#pragma unroll
        for (int lw = 0; lw < C::LW; ++lw)
          asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(wd[kg][lw]) : "r"(kp + (4 * lw + t) * 4));
      } else if constexpr (C::LW == 4) {
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
    // (cell-plane codes: raw over the planes, rawq over the residual signs)
    float raw[4][2], rawq[4][2];
    if constexpr (KR) {
      // rows: keys kb*16 + g (code words wd[2 kb]) and kb*16 + g + 8 (wd[2 kb + 1]);
      // columns 0 / 1: the high / low limb sums; two accumulators per key
      // block (even and odd slices) for independent MMA chains
      // (cell-plane codes: sq for the residual-sign slices, c >= NC_MSE)
      int sc[2][2][4], sq[2][2][4];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int par = 0; par < 2; ++par) {
          sc[kb][par][0] = sc[kb][par][1] = sc[kb][par][2] = sc[kb][par][3] = 0;
          sq[kb][par][0] = sq[kb][par][1] = sq[kb][par][2] = sq[kb][par][3] = 0;
        }
#pragma unroll
      for (int c = 0; c < C::NC; ++c) {
        const int q0 = 2 * c, q1 = 2 * c + 1;
        const int p0 = q0 & 7, p1 = q1 & 7;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const uint32_t wr0 = wd[2 * kb][q0 >> 3], wr8 = wd[2 * kb + 1][q0 >> 3];
          const uint32_t a0 = (wr0 >> p0) & 0x01010101u;
          const uint32_t a1 = (wr8 >> p0) & 0x01010101u;
          const uint32_t a2 = (wr0 >> p1) & 0x01010101u;
          const uint32_t a3 = (wr8 >> p1) & 0x01010101u;
          if (TB > 0 && c >= C::NC_MSE)
            mma_s8_16832(sq[kb][c & 1], a0, a1, a2, a3, bfr[c][0], bfr[c][1]);
          else
            mma_s8_16832(sc[kb][c & 1], a0, a1, a2, a3, bfr[c][0], bfr[c][1]);
        }
      }
      // lane (g, t) holds head t's sum_{bit=1} u_int of keys kb*16 + g
      // (v[kb][0]) and kb*16 + g + 8 (v[kb][1]); head g's key kg*8 + 2t + j
      // sits in lane (2t + j, g)
      int v[2][2], vq[2][2];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        v[kb][0] = (sc[kb][0][0] + sc[kb][1][0]) * 256 + (sc[kb][0][1] + sc[kb][1][1]);
        v[kb][1] = (sc[kb][0][2] + sc[kb][1][2]) * 256 + (sc[kb][0][3] + sc[kb][1][3]);
        vq[kb][0] = (sq[kb][0][0] + sq[kb][1][0]) * 256 + (sq[kb][0][1] + sq[kb][1][1]);
        vq[kb][1] = (sq[kb][0][2] + sq[kb][1][2]) * 256 + (sq[kb][0][3] + sq[kb][1][3]);
      }
#pragma unroll
      for (int kg = 0; kg < 4; ++kg)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int src = (2 * t + j) * 4 + (g & 3);
          const int si = __shfl_sync(0xffffffffu, v[kg >> 1][kg & 1], src);
          raw[kg][j] = hscale[0] * (float)(2 * si - usum[0]);
          if constexpr (TB > 0) {
            const int sj = __shfl_sync(0xffffffffu, vq[kg >> 1][kg & 1], src);
            rawq[kg][j] = hscale[1] * (float)(2 * sj - usum[1]);
          }
        }
      (void)sq;
      (void)vq;
    } else if constexpr (S8) {
      int sc[4][4], sq[4][4];
#pragma unroll
      for (int kg = 0; kg < 4; ++kg) {
        sc[kg][0] = sc[kg][1] = sc[kg][2] = sc[kg][3] = 0;
        sq[kg][0] = sq[kg][1] = sq[kg][2] = sq[kg][3] = 0;
      }
      const int pbase = (C::CODE_BITS >= 128) ? 0 : 4 * (t & 1);
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
          if constexpr (C::CODE_BITS >= 128) {
            w0 = wd[kg][q0 >> 3]; p0 = q0 & 7;
            w1 = wd[kg][q1 >> 3]; p1 = q1 & 7;
          } else {
            w0 = w1 = wd[kg][0]; p0 = pbase + q0; p1 = pbase + q1;
          }
          // bytes j = bits p + 8j: {0, 1} per coordinate
          const uint32_t b0 = (w0 >> p0) & 0x01010101u;
          const uint32_t b1 = (w1 >> p1) & 0x01010101u;
          if (TB > 0 && c >= C::NC_MSE)
            mma_s8_16832(sq[kg], a0, a1, a2, a3, b0, b1);
          else
            mma_s8_16832(sc[kg], a0, a1, a2, a3, b0, b1);
        }
      }
      // sum_i u_i sign_i = hscale * (2 * sum_{bit=1} u_int - sum u_int)
#pragma unroll
      for (int kg = 0; kg < 4; ++kg)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          raw[kg][j] = hscale[0] * (float)(2 * (sc[kg][j] * 256 + sc[kg][j + 2]) - usum[0]);
          if constexpr (TB > 0)
            rawq[kg][j] = hscale[1] * (float)(2 * (sq[kg][j] * 256 + sq[kg][j + 2]) - usum[1]);
        }
    } else {
      float sc[4][4], sq[4][4];
#pragma unroll
      for (int kg = 0; kg < 4; ++kg) sc[kg][0] = sc[kg][1] = sc[kg][2] = sc[kg][3] = 0.f;
      if constexpr (TB > 0) {
#pragma unroll
        for (int kg = 0; kg < 4; ++kg) sq[kg][0] = sq[kg][1] = sq[kg][2] = sq[kg][3] = 0.f;
      }
      const int pbase = (C::CODE_BITS >= 128) ? 0 : 8 * (t & 1);
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
          if constexpr (C::CODE_BITS >= 128) {
            w0 = wd[kg][q0 >> 4]; p0 = q0 & 15;
            w1 = wd[kg][q1 >> 4]; p1 = q1 & 15;
          } else {
            w0 = w1 = wd[kg][0]; p0 = pbase + q0; p1 = pbase + q1;
          }
          const uint32_t b0 = ((w0 << (15 - p0)) & 0x80008000u) ^ 0xBF80BF80u;
          const uint32_t b1 = ((w1 << (15 - p1)) & 0x80008000u) ^ 0xBF80BF80u;
          if (TB > 0 && c >= C::NC_MSE)
            mma_bf16_16816(sq[kg], a0, a1, a2, a3, b0, b1);
          else
            mma_bf16_16816(sc[kg], a0, a1, a2, a3, b0, b1);
        }
      }
#pragma unroll
      for (int kg = 0; kg < 4; ++kg)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          raw[kg][j] = sc[kg][j] + sc[kg][j + 2];
          if constexpr (TB > 0) rawq[kg][j] = sq[kg][j] + sq[kg][j + 2];
        }
    }

    // ---- estimator, masking, online softmax (head g, keys kg*8 + 2t + j)
    float l2[4][2];
    float bmax = -INFINITY;
    constexpr int NG = 16 / C::NORM_BYTES;  // keys per 16-byte norm group
    const uint32_t nrow =
        ring.norm(s) +
        (maps.tma_codes ? 0u : (uint32_t)((kv_base + key0) & (NG - 1)) * C::NORM_BYTES);
#pragma unroll
    for (int kg = 0; kg < 4; ++kg) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = kg * 8 + 2 * t + j;
        float sval;
        if constexpr (TB > 0) {
          // s = ||k|| (<w, c[cell]> + sqrt(pi/2)/m ||rt|| <S w, sign(S rt)>)
          uint32_t nb;
          asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(nb) : "r"(nrow + key * 4));
          const float nk = __half2float(__ushort_as_half((unsigned short)(nb & 0xFFFFu)));
          const float nr = __half2float(__ushort_as_half((unsigned short)(nb >> 16)));
          sval = nk * fmaf(p.coef * nr, rawq[kg][j], raw[kg][j]);
        } else {
          unsigned short hb;
          asm volatile("ld.shared.u16 %0, [%1];\n" : "=h"(hb) : "r"(nrow + key * 2));
          const float nk = __half2float(__ushort_as_half(hb));
          sval = (p.coef * nk) * raw[kg][j];
        }
        l2[kg][j] = sval * p.scale_log2;
        if (p.scores != nullptr && key < nval && g < Gg &&
            JL_IN_RANGE(p.err, ((int64_t)b_idx * p.Hq + hq0 + g) * p.score_stride + key0 + key,
                        1, (int64_t)p.B * p.Hq * p.score_stride))
          p.scores[((int64_t)b_idx * p.Hq + hq0 + g) * p.score_stride + key0 + key] = sval;
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
    if (__any_sync(0xffffffffu, (al0 != 1.f) || (al1 != 1.f))) {
#pragma unroll
      for (int dt = 0; dt < C::DT; ++dt) {
        acc[dt][0] *= al0; acc[dt][1] *= al1;
        acc[dt][2] *= al0; acc[dt][3] *= al1;
      }
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
      issue_block<M, D, S8, PAGED, TB>(p, maps, ring, ipos, s, lane);
      pos_next<PAGED>(p, ipos);
      if constexpr (PAGED) load_page(ipos);
    }
    pos_next<PAGED, false>(p, pos);
  }
  griddep_launch_dependents();
  if (failed) {
    // let the copies already started land before the warp's shared memory
    // goes away: the ring (two stages) holds block i, whose wait ran out, and
    // block i + 1 if it exists; block j sits in stage j % 2 and completes
    // phase (j / 2) & 1 of its barrier
    static_assert(C::STAGES == 2, "drain written for a two-stage ring");
    if (!p.drop_copies) {
      const int j = (failed >> 1) & 3;
      mbar_wait_bounded(ring.bar(j & 1), (uint32_t)(j >> 1), p.wait_ns);
      if (failed & 8)
        mbar_wait_bounded(ring.bar((j + 1) & 1), (uint32_t)(((j + 1) >> 1) & 1), p.wait_ns);
    }
    return;
  }
  if (cur_u >= 0) flush(cur_u);
}

// ---------------------------------------------------------------------------
// 3. combine the partial states of each (b, query head).  Warp 0 reads every
// slot's (max, sum) at once and leaves the slot weights in shared memory; then
// each thread (one output dimension) sums its weighted column with several
// loads in flight.
// one unit can be split over every warp of the launch: at most W_bound + 1
constexpr int COMB_MAX_SLOTS = DEC_SM_COUNT * DEC_MAX_CTAS_SM * DEC_WARPS + 1;

template <int D, bool PAGED>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecParams p,
                                                           uint16_t *__restrict__ out) {
  __shared__ float wts[COMB_MAX_SLOTS];
  __shared__ float inv_l, comb_mx, comb_l;
  __shared__ int64_t red[2][D / 32];
  const float *__restrict__ partials = p.partials;
  const int Hq = p.Hq, G = p.G;
  int W = p.W;
  const int bh = blockIdx.x;
  const int b = bh / Hq, hq = bh - b * Hq;
  const int hkv = hq / G, hl = hq - hkv * G;
  const int hg = hl / DEC_HPAD, hh = hl - hg * DEC_HPAD;
  const int64_t u = ((int64_t)b * p.Hkv + hkv) * p.HG + hg;
  int64_t first, last, NB;
  if constexpr (PAGED) {
    // the unit's blocks in the flat space: those of the sequences before b,
    // then this sequence's units in order (as the scorer's plan)
    int64_t pre = 0, tot = 0;
    for (int bb = threadIdx.x; bb < p.B; bb += D) {
      const int64_t n = paged_blocks(p.seq_lens, bb, p.append, p.T);
      tot += n;
      pre += bb < b ? n : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
      pre += __shfl_xor_sync(0xffffffffu, pre, o);
    }
    if ((threadIdx.x & 31) == 0) {
      red[0][threadIdx.x >> 5] = tot;
      red[1][threadIdx.x >> 5] = pre;
    }
    __syncthreads();
    tot = pre = 0;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      tot += red[0][k];
      pre += red[1][k];
    }
    const int64_t nbs = paged_blocks(p.seq_lens, b, p.append, p.T);
    if (threadIdx.x == 0 && hq == 0) {  // a length outside [0, bound]
      const int64_t len = __ldg(p.seq_lens + b);
      if (len < 0 || len + p.append > p.T) record_device_error(p.err, DERR_DECODE_PLAN);
    }
    if (nbs == 0) {  // nothing to attend over: zeros
      out[(int64_t)bh * D + threadIdx.x] = 0;
      return;
    }
    NB = tot * p.UH;
    first = pre * p.UH + (u - (int64_t)b * p.UH) * nbs;
    last = first + nbs - 1;
    W = (int)(NB < W ? NB : W);  // as the scorer
  } else {
    NB = p.NB;
    first = u * p.nb_u;
    last = (u + 1) * p.nb_u - 1;
  }
  griddep_wait();  // every partial state of the scorer is needed
  const int f = warp_of_block(first, NB, W);
  const int l = warp_of_block(last, NB, W);
  int n = min(l - f + 1, COMB_MAX_SLOTS);
  // the unit's records f + u .. f + u + n - 1 must lie in the workspace
  if (!JL_IN_RANGE(p.err, (int64_t)f + u, n, p.slots)) n = 0;
  // records of unit u: warp w wrote record w + u (see the scorer's flush)
  const float *rec0 = partials + (size_t)((int64_t)f + u) * DEC_HPAD * (D + 2) +
                      (size_t)hh * (D + 2);
  const size_t sstride = (size_t)DEC_HPAD * (D + 2);
  if (threadIdx.x < 32) {
    // (max, sum) of every slot in one round of loads; slots past 32 per lane
    // are rare (one unit spread over more than 32 warps)
    const int lane = threadIdx.x;
    float mx = -INFINITY;
    for (int s = lane; s < n; s += 32) {
      const float ms = rec0[s * sstride + D];
      wts[s] = ms;
      mx = fmaxf(mx, ms);
    }
    const float lsl = lane < n ? rec0[lane * sstride + D + 1] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float L = 0.f;
    for (int s = lane; s < n; s += 32) {
      const float wgt = fast_exp2(wts[s] - mx);
      wts[s] = wgt;
      L = fmaf(wgt, s == lane ? lsl : rec0[s * sstride + D + 1], L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      inv_l = 1.f / L;
      comb_mx = mx;
      comb_l = L;
    }
  }
  __syncthreads();
  const int dim = threadIdx.x;
  // the first 32 slots: every load issued before the first multiply
  float v[32];
#pragma unroll
  for (int s = 0; s < 32; ++s) v[s] = s < n ? rec0[s * sstride + dim] : 0.f;
  float o = 0.f;
#pragma unroll
  for (int s = 0; s < 32; ++s) o = s < n ? fmaf(wts[s], v[s], o) : o;
  for (int s = 32; s < n; ++s) o = fmaf(wts[s], rec0[s * sstride + dim], o);
  if (p.state) {
    // the unit's state as one record of the same form: (acc, max, sum)
    const int64_t at = (int64_t)bh * (D + 2);
    if (JL_IN_RANGE(p.err, at, D + 2, (int64_t)p.B * Hq * (D + 2))) {
      p.state[at + dim] = o;
      if (dim == 0) {
        p.state[at + D] = comb_mx;
        p.state[at + D + 1] = comb_l;
      }
    }
    return;
  }
  if (JL_IN_RANGE(p.err, (int64_t)bh * D + dim, 1, (int64_t)p.B * Hq * D))
    out[(int64_t)bh * D + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(o * inv_l));
}

// ---------------------------------------------------------------------------
// 3b. merge of attention states computed over disjoint parts of one context
// (as the combine leaves them with a state buffer: acc[D], max, sum, softmax
// weights 2^(x - max)).  The same log-sum-exp merge as the combine: every
// part is rescaled to the largest max; parts with no keys (sum 0) drop out,
// and a row with none is zero.  One CTA of D threads per row.
template <int D>
__global__ void __launch_bounds__(D) merge_states_kernel(const float *__restrict__ states,
                                                         int R, int64_t rows,
                                                         uint16_t *__restrict__ out, int *err) {
  const int64_t row = blockIdx.x;
  const int dim = threadIdx.x;
  const size_t pstride = (size_t)rows * (D + 2);
  const float *rec = states + (size_t)row * (D + 2);
  float mx = -INFINITY;
  for (int r = 0; r < R; ++r) {
    const float l = __ldg(rec + r * pstride + D + 1);
    if (l > 0.f) mx = fmaxf(mx, __ldg(rec + r * pstride + D));
  }
  float L = 0.f, o = 0.f;
  if (mx > -INFINITY) {
    for (int r = 0; r < R; ++r) {
      const float l = __ldg(rec + r * pstride + D + 1);
      if (l > 0.f) {
        const float w = fast_exp2(__ldg(rec + r * pstride + D) - mx);
        L = fmaf(w, l, L);
        o = fmaf(w, __ldg(rec + r * pstride + dim), o);
      }
    }
  }
  if (JL_IN_RANGE(err, row * D + dim, 1, rows * D))
    out[row * D + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(L > 0.f ? o / L : 0.f));
}

cudaError_t launch_merge_states(const float *states, int R, int64_t rows, int d,
                                uint16_t *out, cudaStream_t stream) {
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
  if (d == 128)
    merge_states_kernel<128><<<(unsigned)rows, 128, 0, stream>>>(states, R, rows, out, err);
  else if (d == 64)
    merge_states_kernel<64><<<(unsigned)rows, 64, 0, stream>>>(states, R, rows, out, err);
  else
    return cudaErrorNotSupported;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 4. paged calls: one prep launch of 256-thread CTAs does the query
// projections (four queries per CTA) and, when keys are given, appends each
// sequence's new key (four keys per CTA); each group of four is split over
// m / 64 CTAs by sketch rows (blockIdx.y), the first of which also stores
// the key's norm and value row.  The scorer and the combine derive
// the work split from seq_lens themselves.
struct PrepParams {
  const void *Q;
  const uint16_t *S;
  float *U;
  int nq;                       // B * Hq
  const void *K_new;            // B x Hkv x d, nullable
  const uint16_t *V_new;        // B x Hkv x d
  uint32_t *sign_pages;
  uint16_t *norm_pages;
  uint16_t *value_pages;
  int num_pages, page_tokens, max_pages;
  const int32_t *block_table;
  const int32_t *seq_lens;
  int B, Hkv, append;
  int64_t max_len;
  int *err;
};

template <int M, int D, bool QF32, bool KF32>
__global__ void __launch_bounds__(PROJ_THREADS) paged_prep_kernel(const PrepParams pp) {
  __shared__ float ys[PROJ_VECS][M];
  // launched early behind the previous kernel on the stream (programmatic
  // dependent launch): wait for it before reading anything, then let the
  // scorer be scheduled; it waits for this grid's results where it needs them
  griddep_wait();
  griddep_launch_dependents();
  constexpr int RS = proj_splits<M>();  // blockIdx.y: this CTA's rows of S
  const int split = (int)blockIdx.y;
  const int bid = blockIdx.x;
  const int i = threadIdx.x;
  const int qctas = (pp.nq + PROJ_VECS - 1) / PROJ_VECS;
  if (bid < qctas) {
    // ---- query projections u = S q, four queries per CTA
    const int64_t x0 = (int64_t)bid * PROJ_VECS;
    const int nx = (int)min((int64_t)PROJ_VECS, (int64_t)pp.nq - x0);
    project4<M, D, QF32, RS>(pp.S, pp.Q, x0, nx, pp.U + x0 * M, M,
                             ProjLimits{pp.err, (int64_t)pp.nq * D, ((int64_t)pp.nq - x0) * M},
                             split);
    return;
  }
  const int nkv = pp.B * pp.Hkv;
  const int actas = pp.append ? (nkv + PROJ_VECS - 1) / PROJ_VECS : 0;
  if (bid < qctas + actas) {
    // ---- append: quantize keys kvi = b*Hkv + hkv (four per CTA) and store
    // each at position seq_lens[b] of its sequence
    const int x0 = (bid - qctas) * PROJ_VECS;
    const int nx = min(PROJ_VECS, nkv - x0);
    project4<M, D, KF32, RS>(pp.S, pp.K_new, x0, nx, &ys[0][0], M,
                             ProjLimits{pp.err, (int64_t)nkv * D, PROJ_VECS * M}, split);
    __syncthreads();
    const int lane = i & 31, j = i >> 5;  // warp j stores key x0 + j
    if (j >= nx) return;
    const int kvi = x0 + j;
    const int b = kvi / pp.Hkv, hkv = kvi - b * pp.Hkv;
    const int64_t pos = pp.seq_lens[b];
    const int64_t pidx = pos / pp.page_tokens;
    const int page = (pos >= 0 && pidx < pp.max_pages)
                         ? pp.block_table[(int64_t)b * pp.max_pages + pidx] : -1;
    if (page < 0 || page >= pp.num_pages || pos + 1 > pp.max_len) {
      if (lane == 0) record_device_error(pp.err, DERR_DECODE_PLAN);
      return;
    }
    const int64_t slot = ((int64_t)page * pp.Hkv + hkv) * pp.page_tokens + (pos % pp.page_tokens);
    if (!JL_IN_RANGE(pp.err, slot, 1, (int64_t)pp.num_pages * pp.Hkv * pp.page_tokens)) return;
    // this CTA's code words: rows [split * M / RS, (split + 1) * M / RS)
#pragma unroll
    for (int w = split * (M / RS / 32); w < (split + 1) * (M / RS / 32); ++w) {
      // bit l of word w: coordinate 32w + l >= 0
      const uint32_t word = __ballot_sync(0xffffffffu, ys[j][w * 32 + lane] >= 0.f);
      if (lane == 0) pp.sign_pages[slot * (M / 32) + w] = word;
    }
    if (split != 0) return;  // the first split stores the norm and the value row
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) {
      const float x = KF32 ? reinterpret_cast<const float *>(pp.K_new)[(int64_t)kvi * D + c]
                           : bf16_bits_to_f32(
                                 reinterpret_cast<const uint16_t *>(pp.K_new)[(int64_t)kvi * D + c]);
      ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) pp.norm_pages[slot] = __half_as_ushort(__float2half_rn(sqrtf(ss)));
    const uint32_t *vsrc = reinterpret_cast<const uint32_t *>(pp.V_new + (int64_t)kvi * D);
    uint32_t *vdst = reinterpret_cast<uint32_t *>(pp.value_pages + slot * D);
    for (int c = lane; c < D / 2; c += 32) vdst[c] = vsrc[c];
    return;
  }
}

// TurboQuant-prod paged step: the query rows (as turbo_qproj_kernel), then the
// appended keys, four per CTA.  Per key: y = Pi k / ||k|| (the coalesced
// projection routine on the bf16 rotation), its cells by the odd-symmetric
// rule of the tensor-core quantizer (y > 0 picks the side, |y| against the
// positive boundaries the magnitude; a value on a boundary stays inward),
// r = y - c[cell] and ||r||, rt = bf16(r), then S rt (the same routine) and
// its signs.  Plane and sign words come from warp ballots over the
// coordinates.  The products are accumulated in fp32 in another order than
// the tensor-core quantizer's, so a coordinate within that rounding of a
// boundary (or a sign within it of 0) may come out either way.
struct TurboPrepParams {
  PrepParams pp;                // pp.sign_pages holds the full codes
  const uint16_t *Pi;           // d x d bf16
  const float *Pinv;            // d x d fp32
  WalshCoef wc;
  float mag[4];                 // centroid magnitudes (positive half)
  float pos_thr[3];             // positive boundaries between them
};

template <int M, int D, int TB, bool QF32, bool KF32>
__global__ void __launch_bounds__(PROJ_THREADS) turbo_paged_prep_kernel(const TurboPrepParams tp) {
  constexpr int WORDS = (TB * D + M) / 32;
  __shared__ float ys[PROJ_VECS][D];
  __shared__ float rs[PROJ_VECS][D];
  __shared__ float zs[PROJ_VECS][M];
  const PrepParams &pp = tp.pp;
  griddep_wait();
  griddep_launch_dependents();
  const int bid = blockIdx.x;
  const int qctas = (pp.nq + PROJ_VECS - 1) / PROJ_VECS;
  if (bid < qctas) {
    turbo_query_rows<M, D, TB, QF32>(pp.Q, tp.Pinv, pp.S, pp.U, pp.nq, tp.wc,
                                      (int64_t)bid * PROJ_VECS, pp.err);
    return;
  }
  const int nkv = pp.B * pp.Hkv;
  const int x0 = (bid - qctas) * PROJ_VECS;
  if (!pp.append || x0 >= nkv) return;  // uniform over the CTA
  const int nx = min(PROJ_VECS, nkv - x0);
  const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;  // warp j: key x0 + j
  project4<D, D, KF32>(tp.Pi, pp.K_new, x0, nx, &ys[0][0], D,
                       ProjLimits{pp.err, (int64_t)nkv * D, PROJ_VECS * D});
  __syncthreads();
  uint32_t planes[TB][D / 32];
  float nk = 0.f, rn = 0.f;
  if (j < nx) {
    const int kvi = x0 + j;
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) {
      const float x = KF32 ? reinterpret_cast<const float *>(pp.K_new)[(int64_t)kvi * D + c]
                           : bf16_bits_to_f32(
                                 reinterpret_cast<const uint16_t *>(pp.K_new)[(int64_t)kvi * D + c]);
      ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    nk = sqrtf(ss);
    const float inv = nk > 0.f ? 1.f / nk : 0.f;
    float rsq = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      const int i = 32 * w + lane;
      const float y = ys[j][i] * inv;
      const bool top = y > 0.f;
      const float ay = fabsf(y);
      int mu = 0;  // magnitude cell: number of positive boundaries below |y|
      if constexpr (TB == 2) {
        mu = ay > tp.pos_thr[0];
      } else if constexpr (TB == 3) {
        const int hi = ay > tp.pos_thr[1];
        mu = 2 * hi + (ay > (hi ? tp.pos_thr[2] : tp.pos_thr[0]));
      }
      const float amag = tp.mag[mu];
      const float r = top ? y - amag : y + amag;
      rsq = fmaf(r, r, rsq);
      rs[j][i] = bf16_round_f32(r);
      planes[TB - 1][w] = __ballot_sync(0xffffffffu, top);
#pragma unroll
      for (int k = 0; k < TB - 1; ++k)
        planes[k][w] = __ballot_sync(0xffffffffu, (((mu >> k) & 1) != 0) == top);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rsq += __shfl_xor_sync(0xffffffffu, rsq, o);
    rn = sqrtf(rsq);
  } else {
    for (int c = lane; c < D; c += 32) rs[j][c] = 0.f;
  }
  __syncthreads();
  project4<M, D, true>(pp.S, &rs[0][0], 0, nx, &zs[0][0]);
  __syncthreads();
  if (j >= nx) return;
  const int kvi = x0 + j;
  const int b = kvi / pp.Hkv, hkv = kvi - b * pp.Hkv;
  const int64_t pos = pp.seq_lens[b];
  const int64_t pidx = pos / pp.page_tokens;
  const int page = (pos >= 0 && pidx < pp.max_pages)
                       ? pp.block_table[(int64_t)b * pp.max_pages + pidx] : -1;
  if (page < 0 || page >= pp.num_pages || pos + 1 > pp.max_len) {
    if (lane == 0) record_device_error(pp.err, DERR_DECODE_PLAN);
    return;
  }
  const int64_t slot = ((int64_t)page * pp.Hkv + hkv) * pp.page_tokens + (pos % pp.page_tokens);
  if (!JL_IN_RANGE(pp.err, slot, 1, (int64_t)pp.num_pages * pp.Hkv * pp.page_tokens)) return;
  uint32_t *code = pp.sign_pages + slot * WORDS;
#pragma unroll
  for (int w = 0; w < M / 32; ++w) {
    const uint32_t word = __ballot_sync(0xffffffffu, zs[j][w * 32 + lane] >= 0.f);
    if (lane == 0) code[TB * (D / 32) + w] = word;
  }
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < TB; ++k)
#pragma unroll
      for (int w = 0; w < D / 32; ++w) code[k * (D / 32) + w] = planes[k][w];
    reinterpret_cast<uint32_t *>(pp.norm_pages)[slot] =
        (uint32_t)__half_as_ushort(__float2half_rn(nk)) |
        ((uint32_t)__half_as_ushort(__float2half_rn(rn)) << 16);
  }
  const uint32_t *vsrc = reinterpret_cast<const uint32_t *>(pp.V_new + (int64_t)kvi * D);
  uint32_t *vdst = reinterpret_cast<uint32_t *>(pp.value_pages + slot * D);
  for (int c = lane; c < D / 2; c += 32) vdst[c] = vsrc[c];
}

// ---------------------------------------------------------------------------
// planning and launch
static bool supported(int m, int d) {
  return (d == 64 || d == 128) && (m == 64 || m == 128 || m == 256 || m == 512);
}

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Warps are launched one wave at a time (SMs x resident CTAs x 4), never more
// than this bound, which sizes the partial records: W_bound + units of them.
constexpr int64_t DEC_W_BOUND = (int64_t)DEC_SM_COUNT * DEC_MAX_CTAS_SM * DEC_WARPS;

static bool plan_common(int B, int Hq, int Hkv, int64_t T, int m, int d, DecodePlan *pl) {
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv) return false;
  if ((int64_t)B * Hkv >= ((int64_t)1 << 24) || T >= ((int64_t)1 << 31)) return false;
  if (!supported(m, d)) return false;
  DecodePlan p{};
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.T = T; p.m = m; p.d = d;
  p.G = Hq / Hkv;
  p.HG = (p.G + DEC_HPAD - 1) / DEC_HPAD;
  p.units = B * Hkv * p.HG;
  p.nb_u = (T + DEC_KB - 1) / DEC_KB;
  p.NB = (int64_t)p.units * p.nb_u;
  p.W = (int)(p.NB < DEC_W_BOUND ? p.NB : DEC_W_BOUND);
  p.records = p.W + p.units;
  p.u_bytes = round_up((size_t)B * Hq * m * sizeof(float), 256);
  p.partial_bytes = round_up((size_t)p.records * DEC_HPAD * (d + 2) * sizeof(float), 256);
  *pl = p;
  return true;
}

bool make_decode_plan(int B, int Hq, int Hkv, int64_t T, int m, int d, DecodePlan *pl) {
  if (!plan_common(B, Hq, Hkv, T, m, d, pl)) return false;
  pl->total_bytes = pl->u_bytes + pl->partial_bytes;
  return true;
}

bool make_paged_plan(int B, int Hq, int Hkv, int64_t max_len, int m, int d, DecodePlan *pl) {
  // the same scratch as a contiguous call at the bound: the split itself is
  // derived on the device from the lengths and needs no storage
  return make_decode_plan(B, Hq, Hkv, max_len, m, d, pl);
}

// Tensor maps of one call (see DecMaps).
static bool make_maps(DecMaps *mp, const uint16_t *V, const uint32_t *signs,
                      const uint16_t *norms, int64_t units_kv, int64_t T, int m, int d,
                      int code_bytes = 0, int norm_bytes = 2) {
  if (code_bytes == 0) code_bytes = m / 8;
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  {  // values [units][T][d]: 64 columns x 32 rows x 1 unit, 128-byte swizzle
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)units_kv};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)T * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)DEC_KB, 1};
    if (fn(&mp->value, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(V),
           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  mp->tma_codes = 0;
  mp->sign_elem = (DEC_KB * code_bytes / 4 > 256) ? 8 : 4;
  if (T % 8 != 0) return true;  // per-unit rows not 16-byte aligned: cp.async path
  {  // codes [units][T * code_bytes] as 4- or 8-byte elements, one block per box
    const int es = mp->sign_elem;
    cuuint64_t dims[2] = {(cuuint64_t)(T * code_bytes / es), (cuuint64_t)units_kv};
    cuuint64_t strides[1] = {(cuuint64_t)T * code_bytes};
    cuuint32_t box[2] = {(cuuint32_t)(DEC_KB * code_bytes / es), 1};
    if (fn(&mp->sign, es == 8 ? CU_TENSOR_MAP_DATA_TYPE_UINT64 : CU_TENSOR_MAP_DATA_TYPE_UINT32,
           2, const_cast<uint32_t *>(signs), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return true;
  }
  {  // norms [units][T] binary16 (or binary16 pairs as 4-byte elements), 32 per box
    cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)units_kv};
    cuuint64_t strides[1] = {(cuuint64_t)T * norm_bytes};
    cuuint32_t box[2] = {(cuuint32_t)DEC_KB, 1};
    if (fn(&mp->norm,
           norm_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
           const_cast<uint16_t *>(norms), dims,
           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return true;
  }
  mp->tma_codes = 1;
  return true;
}

// Scoring MMA for a shape: int8 (half the sign-expansion work and MMAs per
// key) unless a bf16 build is forced; see the measurements in the design
// notes for the per-shape choice.
static bool decode_use_s8(int G, int m) {
  if (JL_DECODE_SCORE == 1) return false;
  if (JL_DECODE_SCORE == 2) return true;
  return G == 1 || m > 256;
}

// The keys-as-rows int8 scoring (m >= 128, at most four heads per KV head).
// Measured against the head-rows form on one box (B = 8, T = 32768):
//   G = 1: faster for m >= 4d, slightly slower at m = 2d;
//   G = 4: d = 128, m = 512: 137.5 -> 120.7 us; m = 256: 113.0 -> 115.0 us
//          (slower); m = 128: 106.4 -> 105 us; d = 64, m = 128 / 256 / 512:
//          75.2 -> 71.2, 102.0 -> 77.4, 108.0 -> 104.0 us.
static bool decode_use_keyrows(int G, int m, int d) {
  if (JL_DECODE_SCORE == 1 || m < 128) return false;
  if (G == 1) return m >= 4 * d;
  return G <= 4 && (m >= 4 * d || d == 64);
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

static void fill_params(DecParams &p, const DecodePlan &pl, float *U, float *partials,
                        const uint32_t *signs, const uint16_t *norms, float *scores,
                        float softmax_scale, int m, int *err) {
  p = DecParams{};
  p.U = U; p.signs = signs; p.norms = norms; p.partials = partials;
  p.scores = scores; p.err = err; p.T = pl.T; p.nb_u = pl.nb_u; p.NB = pl.NB;
  p.n_keys = (int64_t)pl.B * pl.Hkv * pl.T;
  p.Hq = pl.Hq; p.Hkv = pl.Hkv; p.G = pl.G; p.HG = pl.HG;
  p.slots = pl.records;
  p.coef = (float)(sqrt(M_PI / 2.0) / (double)m);
  p.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634074);
  p.score_stride = pl.T;
  p.units = pl.units;
  p.B = pl.B;
  p.UH = pl.Hkv * pl.HG;
  p.wait_ns = wait_limit_ns();
  p.drop_copies = 0;
  p.state = nullptr;
}

// Launch the scorer (one wave, <= the plan's warp bound) and the combine.
template <int M, int D, bool S8, bool PAGED, int TB = 0, bool KR = false>
static cudaError_t launch_scorer_combine(const DecodePlan &pl, DecParams &p, const DecMaps &maps,
                                         uint16_t *out, cudaStream_t stream) {
  using C = DecCfg<M, D, S8, TB>;
  auto kern = decode_scorer_kernel<M, D, S8, PAGED, TB, KR>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::CTA_BYTES);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, DEC_WARPS * 32,
                                                    C::CTA_BYTES);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  if (per_sm > DEC_MAX_CTAS_SM) per_sm = DEC_MAX_CTAS_SM;
  const int64_t wave = (int64_t)device_sm_count() * per_sm * DEC_WARPS;
  p.W = (int)(wave < pl.W ? wave : pl.W);
  const int ctas = (p.W + DEC_WARPS - 1) / DEC_WARPS;
  e = launch_pdl(kern, dim3(ctas), dim3(DEC_WARPS * 32), C::CTA_BYTES, stream, maps, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_combine_kernel<D, PAGED>, dim3(pl.B * pl.Hq), dim3(D), 0, stream,
                    (const DecParams)p, out);
}

template <int M, int D, bool S8>
static cudaError_t launch_decode_t(const DecodePlan &pl, const void *Q,
                                   bool q_f32, const uint16_t *S,
                                   const uint32_t *signs, const uint16_t *norms,
                                   const uint16_t *V, float softmax_scale,
                                   uint16_t *out, float *scores,
                                   void *workspace, cudaStream_t stream, float *state) {
  float *U = reinterpret_cast<float *>(workspace);
  float *partials =
      reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + pl.u_bytes);
  DecMaps maps;
  if (!make_maps(&maps, V, signs, norms, (int64_t)pl.B * pl.Hkv, pl.T, M, D))
    return cudaErrorInvalidValue;
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
  const int bh = pl.B * pl.Hq;
  const int qctas = (bh + PROJ_VECS - 1) / PROJ_VECS;
  if (q_f32)
    qproj_kernel<M, D, true><<<dim3(qctas, proj_splits<M>()), PROJ_THREADS, 0, stream>>>(Q, S, U,
                                                                                        bh, err);
  else
    qproj_kernel<M, D, false><<<dim3(qctas, proj_splits<M>()), PROJ_THREADS, 0, stream>>>(Q, S, U,
                                                                                         bh, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DecParams p;
  fill_params(p, pl, U, partials, signs, norms, scores, softmax_scale, M, err);
  p.drop_copies = test_drop_copies() ? 1 : 0;
  p.state = state;
  // one head per KV head and a code at least twice the value row's bytes
  // (m >= 4d): the keys-as-rows int8 scoring (half the MMAs; measured faster
  // there, slightly slower at m = 2d)
  if constexpr (M >= 128) {
    if (decode_use_keyrows(pl.G, M, D))
      return launch_scorer_combine<M, D, true, false, 0, true>(pl, p, maps, out, stream);
  }
  return launch_scorer_combine<M, D, S8, false>(pl, p, maps, out, stream);
}

bool make_turbo_decode_plan(int B, int Hq, int Hkv, int64_t T, int m, int d, int bits,
                            DecodePlan *pl) {
  if (!((m == 128 && d == 128) || (m == 64 && d == 64)) || bits < 1 || bits > 3) return false;
  if (!plan_common(B, Hq, Hkv, T, m, d, pl)) return false;
  const int terms = bits == 3 ? 4 : bits;
  const size_t row = (size_t)(terms * d + 127) / 128 * 128 + (size_t)(m + 127) / 128 * 128;
  pl->u_bytes = round_up((size_t)B * Hq * row * sizeof(float), 256);
  pl->total_bytes = pl->u_bytes + pl->partial_bytes;
  return true;
}

// Scoring MMA of the cell-plane codes: int8 (k = 32 coordinates per MMA,
// four coordinates per expanded register) unless a bf16 build is forced.
constexpr bool TURBO_S8 = JL_DECODE_SCORE != 1;

// Keys-as-rows scoring of cell-plane codes (at most four heads per KV head;
// two accumulator sets and two scales per head, planes and residual signs).
// Measured against the head-rows form on one box (G = 4, B = 8, T = 32768,
// b-1 = 2): d = 128 119.8 -> 116.0 us, d = 64 82.5 -> 77.5 us; the paged
// step within noise (114.5 -> 111.0 / 115.3 us).
static bool turbo_use_keyrows(int G) { return G <= 4; }

template <int TB, int D>
static cudaError_t launch_turbo_decode_t(const DecodePlan &pl, const void *Q, bool q_f32,
                                         const float *Pinv, const uint16_t *S,
                                         const uint32_t *codes, const uint16_t *norms,
                                         const uint16_t *V, const double *walsh,
                                         float softmax_scale, uint16_t *out, float *scores,
                                         void *workspace, cudaStream_t stream) {
  constexpr int M = D;
  float *U = reinterpret_cast<float *>(workspace);
  float *partials =
      reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + pl.u_bytes);
  DecMaps maps;
  if (!make_maps(&maps, V, codes, norms, (int64_t)pl.B * pl.Hkv, pl.T, M, D,
                 DecCfg<M, D, TURBO_S8, TB>::KEY_SIGN_BYTES, 4))
    return cudaErrorInvalidValue;
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
  const int bh = pl.B * pl.Hq;
  const int qctas = (bh + PROJ_VECS - 1) / PROJ_VECS;
  WalshCoef wc;
  for (int k = 0; k < 4; ++k) wc.c[k] = (float)walsh[k];
  if (q_f32)
    turbo_qproj_kernel<M, D, TB, true><<<qctas, PROJ_THREADS, 0, stream>>>(Q, Pinv, S, U, bh, wc,
                                                                            err);
  else
    turbo_qproj_kernel<M, D, TB, false><<<qctas, PROJ_THREADS, 0, stream>>>(Q, Pinv, S, U, bh, wc,
                                                                             err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DecParams p;
  fill_params(p, pl, U, partials, codes, norms, scores, softmax_scale, M, err);
  if (TURBO_S8 && turbo_use_keyrows(pl.G))
    return launch_scorer_combine<M, D, true, false, TB, true>(pl, p, maps, out, stream);
  return launch_scorer_combine<M, D, TURBO_S8, false, TB>(pl, p, maps, out, stream);
}

cudaError_t launch_turbo_decode(const DecodePlan &pl, int bits, const void *Q, bool q_f32,
                                const float *Pinv, const uint16_t *S, const uint32_t *codes,
                                const uint16_t *norms, const uint16_t *V, const double *walsh,
                                float softmax_scale, uint16_t *out, float *scores,
                                void *workspace, cudaStream_t stream) {
#define JL_CASE(TB, DD)                                                                   \
  if (bits == TB && pl.d == DD && pl.m == DD)                                              \
    return launch_turbo_decode_t<TB, DD>(pl, Q, q_f32, Pinv, S, codes, norms, V, walsh,     \
                                         softmax_scale, out, scores, workspace, stream);
  JL_CASE(1, 128) JL_CASE(2, 128) JL_CASE(3, 128) JL_CASE(1, 64) JL_CASE(2, 64) JL_CASE(3, 64)
#undef JL_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_query_projection(const void *Q, bool q_f32, const uint16_t *S, float *U,
                                    int nq, int m, int d, cudaStream_t stream) {
  if (nq <= 0) return cudaSuccess;
  const int ctas = (nq + PROJ_VECS - 1) / PROJ_VECS;
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
#define JL_CASE(MM, DD)                                                                  \
  if (m == MM && d == DD) {                                                              \
    const dim3 grid(ctas, proj_splits<MM>());                                            \
    if (q_f32)                                                                           \
      qproj_kernel<MM, DD, true><<<grid, PROJ_THREADS, 0, stream>>>(Q, S, U, nq, err);    \
    else                                                                                 \
      qproj_kernel<MM, DD, false><<<grid, PROJ_THREADS, 0, stream>>>(Q, S, U, nq, err);   \
    return cudaGetLastError();                                                           \
  }
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_decode(const DecodePlan &pl, const void *Q, bool q_f32,
                          const uint16_t *S, const uint32_t *signs,
                          const uint16_t *norms, const uint16_t *V,
                          float softmax_scale, uint16_t *out, float *scores,
                          void *workspace, cudaStream_t stream, float *state) {
  const bool s8 = decode_use_s8(pl.G, pl.m);
#define JL_CASE(MM, DD)                                                         \
  if (pl.m == MM && pl.d == DD)                                                 \
    return s8 ? launch_decode_t<MM, DD, true>(pl, Q, q_f32, S, signs, norms, V, \
                                              softmax_scale, out, scores,       \
                                              workspace, stream, state)         \
              : launch_decode_t<MM, DD, false>(pl, Q, q_f32, S, signs, norms, V, \
                                               softmax_scale, out, scores,      \
                                               workspace, stream, state);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

// Paged pools: values [num_pages*Hkv][P][d], codes [num_pages*Hkv][P*m/8 bytes],
// norms [num_pages*Hkv][P]; every block is one box inside one page.
static bool make_paged_maps(DecMaps *mp, const PagedArgs &a, int Hkv, int m, int d,
                            int code_bytes = 0, int norm_bytes = 2) {
  if (code_bytes == 0) code_bytes = m / 8;
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  const uint64_t rows = (uint64_t)a.num_pages * Hkv, P = (uint64_t)a.page_tokens;
  {
    cuuint64_t dims[3] = {(cuuint64_t)d, P, rows};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, P * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)DEC_KB, 1};
    if (fn(&mp->value, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.value_pages, dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  mp->sign_elem = (DEC_KB * code_bytes / 4 > 256) ? 8 : 4;
  {
    const int es = mp->sign_elem;
    cuuint64_t dims[2] = {(cuuint64_t)(P * code_bytes / es), rows};
    cuuint64_t strides[1] = {(cuuint64_t)(P * code_bytes)};
    cuuint32_t box[2] = {(cuuint32_t)(DEC_KB * code_bytes / es), 1};
    if (fn(&mp->sign, es == 8 ? CU_TENSOR_MAP_DATA_TYPE_UINT64 : CU_TENSOR_MAP_DATA_TYPE_UINT32,
           2, a.sign_pages, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    cuuint64_t dims[2] = {P, rows};
    cuuint64_t strides[1] = {P * norm_bytes};
    cuuint32_t box[2] = {(cuuint32_t)DEC_KB, 1};
    if (fn(&mp->norm,
           norm_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
           a.norm_pages, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  mp->tma_codes = 1;
  return true;
}

template <int M, int D, bool S8>
static cudaError_t launch_paged_t(const DecodePlan &pl, const PagedArgs &a,
                                  cudaStream_t stream) {
  uint8_t *ws = reinterpret_cast<uint8_t *>(a.workspace);
  float *U = reinterpret_cast<float *>(ws);
  float *partials = reinterpret_cast<float *>(ws + pl.u_bytes);
  DecMaps maps;
  if (!make_paged_maps(&maps, a, pl.Hkv, M, D)) return cudaErrorInvalidValue;
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
  PrepParams pp;
  pp.Q = a.Q; pp.S = a.S; pp.U = U; pp.nq = pl.B * pl.Hq;
  pp.K_new = a.K_new; pp.V_new = a.V_new;
  pp.sign_pages = a.sign_pages; pp.norm_pages = a.norm_pages; pp.value_pages = a.value_pages;
  pp.num_pages = a.num_pages; pp.page_tokens = a.page_tokens; pp.max_pages = a.max_pages;
  pp.block_table = a.block_table; pp.seq_lens = a.seq_lens;
  pp.B = pl.B; pp.Hkv = pl.Hkv;
  pp.append = a.K_new != nullptr;
  pp.max_len = pl.T;
  pp.err = err;
  const int nkv = pl.B * pl.Hkv;
  const int prep_ctas = (pp.nq + PROJ_VECS - 1) / PROJ_VECS +
                        (pp.append ? (nkv + PROJ_VECS - 1) / PROJ_VECS : 0);
  const dim3 pg(prep_ctas, proj_splits<M>()), pb(PROJ_THREADS);
  cudaError_t e;
  if (a.q_f32)
    e = a.k_f32 ? launch_pdl(paged_prep_kernel<M, D, true, true>, pg, pb, 0, stream, pp)
                : launch_pdl(paged_prep_kernel<M, D, true, false>, pg, pb, 0, stream, pp);
  else
    e = a.k_f32 ? launch_pdl(paged_prep_kernel<M, D, false, true>, pg, pb, 0, stream, pp)
                : launch_pdl(paged_prep_kernel<M, D, false, false>, pg, pb, 0, stream, pp);
  if (e != cudaSuccess) return e;
  DecParams p;
  fill_params(p, pl, U, partials, nullptr, nullptr, a.scores, a.softmax_scale, M, err);
  p.seq_lens = a.seq_lens; p.block_table = a.block_table;
  p.max_pages = a.max_pages; p.page_tokens = a.page_tokens; p.append = pp.append;
  p.score_stride = pl.T;
  if constexpr (M >= 128) {  // as the contiguous call
    if (decode_use_keyrows(pl.G, M, D))
      return launch_scorer_combine<M, D, true, true, 0, true>(pl, p, maps, a.out, stream);
  }
  return launch_scorer_combine<M, D, S8, true>(pl, p, maps, a.out, stream);
}

template <int TB, int D>
static cudaError_t launch_turbo_paged_t(const DecodePlan &pl, const PagedArgs &a,
                                        const TurboPagedArgs &t, cudaStream_t stream) {
  constexpr int M = D;
  uint8_t *ws = reinterpret_cast<uint8_t *>(a.workspace);
  float *U = reinterpret_cast<float *>(ws);
  float *partials = reinterpret_cast<float *>(ws + pl.u_bytes);
  DecMaps maps;
  if (!make_paged_maps(&maps, a, pl.Hkv, M, D, DecCfg<M, D, TURBO_S8, TB>::KEY_SIGN_BYTES, 4))
    return cudaErrorInvalidValue;
  int *err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidSymbol;
  TurboPrepParams tp;
  PrepParams &pp = tp.pp;
  pp.Q = a.Q; pp.S = a.S; pp.U = U; pp.nq = pl.B * pl.Hq;
  pp.K_new = a.K_new; pp.V_new = a.V_new;
  pp.sign_pages = a.sign_pages; pp.norm_pages = a.norm_pages; pp.value_pages = a.value_pages;
  pp.num_pages = a.num_pages; pp.page_tokens = a.page_tokens; pp.max_pages = a.max_pages;
  pp.block_table = a.block_table; pp.seq_lens = a.seq_lens;
  pp.B = pl.B; pp.Hkv = pl.Hkv;
  pp.append = a.K_new != nullptr;
  pp.max_len = pl.T;
  pp.err = err;
  tp.Pi = t.Pi;
  tp.Pinv = t.Pinv;
  for (int k = 0; k < 4; ++k) {
    tp.wc.c[k] = (float)t.walsh[k];
    tp.mag[k] = t.mag[k];
  }
  for (int k = 0; k < 3; ++k) tp.pos_thr[k] = t.pos_thr[k];
  const int nkv = pl.B * pl.Hkv;
  const int prep_ctas = (pp.nq + PROJ_VECS - 1) / PROJ_VECS +
                        (pp.append ? (nkv + PROJ_VECS - 1) / PROJ_VECS : 0);
  const dim3 pg(prep_ctas), pb(PROJ_THREADS);
  cudaError_t e;
  if (a.q_f32)
    e = a.k_f32 ? launch_pdl(turbo_paged_prep_kernel<M, D, TB, true, true>, pg, pb, 0, stream, tp)
                : launch_pdl(turbo_paged_prep_kernel<M, D, TB, true, false>, pg, pb, 0, stream, tp);
  else
    e = a.k_f32 ? launch_pdl(turbo_paged_prep_kernel<M, D, TB, false, true>, pg, pb, 0, stream, tp)
                : launch_pdl(turbo_paged_prep_kernel<M, D, TB, false, false>, pg, pb, 0, stream, tp);
  if (e != cudaSuccess) return e;
  DecParams p;
  fill_params(p, pl, U, partials, nullptr, nullptr, a.scores, a.softmax_scale, M, err);
  p.seq_lens = a.seq_lens; p.block_table = a.block_table;
  p.max_pages = a.max_pages; p.page_tokens = a.page_tokens; p.append = pp.append;
  p.score_stride = pl.T;
  if (TURBO_S8 && turbo_use_keyrows(pl.G))
    return launch_scorer_combine<M, D, true, true, TB, true>(pl, p, maps, a.out, stream);
  return launch_scorer_combine<M, D, TURBO_S8, true, TB>(pl, p, maps, a.out, stream);
}

cudaError_t launch_turbo_decode_paged(const DecodePlan &pl, int bits, const PagedArgs &a,
                                      const TurboPagedArgs &t, cudaStream_t stream) {
#define JL_CASE(TB, DD) \
  if (bits == TB && pl.d == DD && pl.m == DD) return launch_turbo_paged_t<TB, DD>(pl, a, t, stream);
  JL_CASE(1, 128) JL_CASE(2, 128) JL_CASE(3, 128) JL_CASE(1, 64) JL_CASE(2, 64) JL_CASE(3, 64)
#undef JL_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_decode_paged(const DecodePlan &pl, const PagedArgs &a,
                                cudaStream_t stream) {
  const bool s8 = decode_use_s8(pl.G, pl.m);
#define JL_CASE(MM, DD)                                            \
  if (pl.m == MM && pl.d == DD)                                    \
    return s8 ? launch_paged_t<MM, DD, true>(pl, a, stream)        \
              : launch_paged_t<MM, DD, false>(pl, a, stream);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
