// search_tc.cu -- inner-product top-k search over a QJL-compressed index.
//
// "The Geometry of Forgetting: How Three Papers Cracked KV Cache
// Quantization", final section: the quantizer serves any store of
// high-dimensional vectors that is read through inner products (vector
// databases, retrieval, recommendation).  Here each index vector x is kept as
// its QJL code z = sign(S x) and norm, and a query q is scored against every
// vector with the asymmetric estimator of the QJL section,
//     s(q, x) = sqrt(pi/2)/m * ||x|| * <S q, z>,
// keeping the k best vectors per query.
//
// One pass handles up to 128 queries.  For a tile of 256 index vectors the
// scores form a dense contraction D[128 queries][256 vectors] = U Z^T
// (M = 128, N = 256, K = m) on the tensor cores:
//   * U = S q (projected by the query-projection kernel) is rounded to fp16
//     with a power-of-two scale per query (relative error <= 2^-11 per
//     coordinate) and written once as the A operand: into shared memory
//     (128-byte swizzle, K-major) for m <= 256, so that tensor memory holds
//     two accumulators and the MMAs of one tile overlap the epilogue of the
//     previous one; into tensor memory beside a single accumulator for
//     m = 512;
//   * the B operand is Z scaled by each vector's norm, +-||x|| in fp16 (the
//     norms are stored in binary16, and a product with the fp16 U is exact
//     in fp32), expanded from the code bits into shared memory one K-chunk of
//     64 coordinates (32 KB) at a time: an fp16 pair holds coordinates
//     (p, p + 16) of a code word, ((w << (15 - p)) & 0x80008000) ^
//     (0x80008000 | ||x|| ||x||), and U's columns use the same order;
//   * each accumulator takes 256 fp32 columns of tensor memory.  (An MMA of
//     N = 128 runs at about two thirds of the rate per flop of N = 256 here,
//     so the tile stays 256 wide.)
// Each epilogue lane owns one query and keeps its best KT scores (before the
// query's positive output scale) in registers.  Per 32 columns the hot path
// is the group maximum and one comparison with the list's bound: the larger
// of the list's own KT-th best and the best KT-th best any list of the query
// has published so far (a lower bound on the final KT-th best, shared
// through an atomic maximum in global memory).  Only a lane whose group
// passes parks its 32 scores in a private row of shared memory and inserts
// the qualifying ones.  A second kernel merges the lists of each query.
// Before the full pass, the same kernel scores the queries against a spread
// sample of the index tiles, and the merge kernel turns each query's 16th
// best sample score into its starting bound (a valid lower bound on the
// final 16th best: the sample is part of the index), so that very few scores
// of the full pass reach the insertion path.
//
// One persistent CTA per SM, 9 warps with fixed roles:
//   warps 0-3  expand: thread t owns rows t and t + 128 of every tile.
//   warps 4-7  U into tensor memory first, then the epilogue: lane quadrant
//              warp % 4 = queries 32 (warp % 4) .. + 31, one list per query.
//   warp 8     owns the TMEM allocation; the whole warp runs the MMA loop
//              and one elected lane issues the MMAs (descriptors are
//              precomputed: an operand is the base plus a 32-bit add).
// Every mbarrier wait is bounded; a wait that runs out records
// DERR_TC_WAIT_TIMEOUT and the CTA still frees its TMEM.
#include "jl_common.cuh"
#include "jl_internal.h"
#include "jl_tc.cuh"

#include <math.h>

namespace jlk {
namespace srch {

using namespace tcx;

constexpr int QM = 128;                        // queries per pass (MMA M)
constexpr int BN = 256;                        // index vectors per tile (MMA N)
constexpr int CHUNK_K = 64;                    // coordinates per Z chunk
constexpr int CHUNK_BYTES = BN * CHUNK_K * 2;  // 32 KB
constexpr int EXP_WARPS = 4, EPI_WARPS = 4;
constexpr int LISTS = 1;                       // lists per query and CTA
constexpr int PARK_ROWS = 2;                   // groups a lane can park at once
constexpr int MMA_WARP = EXP_WARPS + EPI_WARPS;
constexpr int THREADS = (MMA_WARP + 1) * 32;
constexpr int CODE_SLOTS = 3;
constexpr int TMEM_COLS = 512;
constexpr int MAX_CTAS = 256;                  // bounds the per-CTA lists
constexpr int MERGE_THREADS = 256;

template <int M>
struct Cfg {
  static constexpr int KCH = M / CHUNK_K;
  static constexpr bool U_SMEM = M <= 256;     // A operand in shared memory
  static constexpr int U_COLS = U_SMEM ? 0 : M / 2;  // tensor-memory columns of U (fp16 pairs)
  static constexpr int NACC = U_SMEM ? 2 : 1;  // accumulators of BN columns
  static constexpr int D_COL = U_COLS;         // accumulator b: columns D_COL + BN b ...
  static constexpr int RING = 3;
  static constexpr int CODE_ROW = M / 8;
  static constexpr int CODE_WORDS = M / 32;
  static constexpr int U_CHUNK = QM * 128;     // one 64-coordinate K-chunk of U
  static constexpr int OFF_U = 0;
  static constexpr int OFF_Z = OFF_U + (U_SMEM ? KCH * U_CHUNK : 0);
  static constexpr int OFF_C = OFF_Z + RING * CHUNK_BYTES;
  // per epilogue lane: PARK_ROWS rows of 33 floats (parked groups)
  static constexpr int OFF_P = OFF_C + CODE_SLOTS * BN * CODE_ROW;
  static constexpr int OFF_BAR = OFF_P + EPI_WARPS * 32 * PARK_ROWS * 33 * 4;
  static constexpr int NBAR = 2 * RING + 2 * NACC;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static_assert(D_COL + NACC * BN <= TMEM_COLS, "tensor memory columns");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct Params {
  const uint32_t *signs;   // N x m/32
  const uint16_t *norms;   // N binary16
  const float *U;          // QM x m (rows >= nq ignored)
  float *part_val;         // [MAX_CTAS][LISTS][QM][KT]
  int32_t *part_idx;
  unsigned *gbound;        // [QM] order-preserving codes of the shared bounds (0 = none)
  float *qscale;           // [QM] output scale of each query's scores
  int64_t N;
  int64_t num_tiles;       // tiles of this launch: tile0 + j * tile_step, j < num_tiles
  int64_t tile0, tile_step;
  int nq;
  float coef;              // sqrt(pi/2) / m
  int *err;
};



// Copy code rows `row0` and `row0 + 128` (M/8 bytes each) into shared memory
// with cp.async, zero fill past the end, as one commit group.
template <int M>
__device__ __forceinline__ void copy_code_rows(uint32_t dst0, uint32_t dst1, const uint32_t *signs,
                                               int64_t row0, int64_t N, int *err) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t row = row0 + 128 * h;
    const bool live = row < N && JL_IN_RANGE(err, row * (M / 8), M / 8, N * (M / 8));
    const uint32_t dst = h ? dst1 : dst0;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(signs + (live ? row : 0) * (M / 32));
    if constexpr (M >= 128) {
#pragma unroll
      for (int q = 0; q < M / 128; ++q) cp_async_16(dst + 16 * q, src + 16 * q, live ? 16 : 0);
    } else {
      cp_async_8(dst, src, live ? 8 : 0);
    }
  }
  cp_async_commit();
}

// Expand two 32-bit code words into one 128-byte row of a B chunk (fp16
// +-||x||, pair j of word h at 16-byte unit 4 h + j / 4), swizzled by
// (row & 7); x = 0x80008000 | the norm's bits in both halves.
__device__ __forceinline__ void expand_row(uint8_t *chunk, int r, uint32_t w0, uint32_t w1,
                                           uint32_t x) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t w = half ? w1 : w0;
#pragma unroll
    for (int u4 = 0; u4 < 4; ++u4) {
      uint32_t q[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * u4 + e;
        q[e] = ((w << (15 - j)) & 0x80008000u) ^ x;
      }
      const int unit = 4 * half + u4;
      *reinterpret_cast<uint4 *>(chunk + r * 128 + ((unit ^ (r & 7)) << 4)) =
          make_uint4(q[0], q[1], q[2], q[3]);
    }
  }
}

// max(a, b, c) in one instruction (three-input max.f32)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Order-preserving code of a float (larger float <-> larger code; never 0 for
// a number), and back.
__device__ __forceinline__ unsigned ord_code(float f) {
  const unsigned b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_float(unsigned c) {
  if (c == 0u) return -INFINITY;
  return __uint_as_float((c & 0x80000000u) ? (c & 0x7FFFFFFFu) : ~c);
}

// A query's list of its KT best (score, index): filled in order, then the
// minimum is replaced.  All indexing is static so the list stays in registers.
template <int KT>
struct TopList {
  float val[KT];
  int32_t idx[KT];
  int cnt;
  float thr;  // the smallest kept score once the list is full, else -inf

  __device__ __forceinline__ void init() {
    cnt = 0;
    thr = -INFINITY;
#pragma unroll
    for (int e = 0; e < KT; ++e) {
      val[e] = -INFINITY;
      idx[e] = -1;
    }
  }
  __device__ __forceinline__ float min_val() const {
    float mv = val[0];
#pragma unroll
    for (int e = 1; e < KT; ++e) mv = fminf(mv, val[e]);
    return mv;
  }
  __device__ __forceinline__ void insert(float s, int32_t i) {
    if (cnt < KT) {
#pragma unroll
      for (int e = 0; e < KT; ++e)
        if (e == cnt) {
          val[e] = s;
          idx[e] = i;
        }
      if (++cnt == KT) thr = min_val();
    } else {
      bool done = false;
#pragma unroll
      for (int e = 0; e < KT; ++e)
        if (!done && val[e] == thr) {
          val[e] = s;
          idx[e] = i;
          done = true;
        }
      thr = min_val();
    }
  }
};

// --------------------------------------------------------------------------
template <int M, int KT>
__global__ void __launch_bounds__(THREADS, 1) search_tc_kernel(const Params p) {
  using C = Cfg<M>;
  extern __shared__ uint8_t sr_smem_raw[];
  const uint32_t raw = smem_u32(sr_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = sr_smem_raw + (base - raw);
  const uint32_t sZ = base + C::OFF_Z;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto zfull_bar = [&](int s) { return bar0 + 8u * s; };
  auto zempty_bar = [&](int s) { return bar0 + 8u * (C::RING + s); };
  auto dfull_bar = [&](int b) { return bar0 + 8u * (2 * C::RING + b); };
  auto dempty_bar = [&](int b) { return bar0 + 8u * (2 * C::RING + C::NACC + b); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int *abort_flag =
      reinterpret_cast<volatile int *>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::RING; ++s) {
      mbar_init(zfull_bar(s), EXP_WARPS);
      mbar_init(zempty_bar(s), 1);
    }
    for (int b = 0; b < C::NACC; ++b) {
      mbar_init(dfull_bar(b), 1);
      mbar_init(dempty_bar(b), EPI_WARPS);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
        "tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::"r"(
            smem_u32(tmem_holder)),
        "n"(TMEM_COLS)
        : "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // ---- U (warps 4-7, query qi = 32 (warp % 4) + lane): fp16 pairs
  // (u_{32b+j}, u_{32b+j+16}) as K positions 2 c, 2 c + 1 with c = 16 b + j,
  // scaled by 2^e per query; into shared memory (word c of row qi in the
  // swizzled K-chunk c / 32) or tensor memory (column c of lane qi)
  if (warp >= EXP_WARPS && warp < MMA_WARP) {
    const int q = warp & 3;
    const int qi = 32 * q + lane;
    const bool valid = qi < p.nq;
    const float *urow = p.U + (int64_t)(valid ? qi : 0) * M;
    float mx = 0.f;
    if (valid)
      for (int i = 0; i < M; ++i) mx = fmaxf(mx, fabsf(urow[i]));
    int ex = 0;
    if (mx > 0.f) frexpf(mx, &ex);          // mx = f 2^ex, f in [0.5, 1)
    const float scale = ldexpf(1.f, 15 - ex);  // max |u| scale in [2^14, 2^15)
    // output scale of the query's scores: sqrt(pi/2)/m * 2^-e
    if (blockIdx.x == 0) p.qscale[qi] = p.coef * ldexpf(1.f, ex - 15);
#pragma unroll 1
    for (int c0 = 0; c0 < M / 2; c0 += 32) {
      uint32_t v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int c = c0 + e, b = c >> 4, j = c & 15;
        const float lo = valid ? urow[32 * b + j] * scale : 0.f;
        const float hi = valid ? urow[32 * b + j + 16] * scale : 0.f;
        __half2 h = __floats2half2_rn(lo, hi);
        v[e] = *reinterpret_cast<uint32_t *>(&h);
      }
      if constexpr (C::U_SMEM) {
        // 32 words = one 128-byte row of K-chunk c0 / 32: eight 16-byte units
        uint8_t *rowp = gbase + C::OFF_U + (c0 / 32) * C::U_CHUNK + qi * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4 *>(rowp + ((u ^ (qi & 7)) << 4)) =
              make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
      } else {
        st32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
      }
    }
    if constexpr (C::U_SMEM) fence_async_smem();
    else st_wait();
  }
  fence_before();
  __syncthreads();
  fence_after();

  const int64_t ntiles = p.num_tiles;
  auto tile_at = [&](int64_t j) { return p.tile0 + j * p.tile_step; };  // rows past N: zero codes
  if (warp < EXP_WARPS) {
    // ---------------- expand: rows t and t + 128 of every tile
    const int t = threadIdx.x;
    const uint32_t crow0 = base + C::OFF_C + t * C::CODE_ROW;
    auto slot0 = [&](int slot) { return crow0 + (uint32_t)(slot * BN * C::CODE_ROW); };
    for (int k = 0; k < CODE_SLOTS - 1; ++k) {
      const int64_t row0 = tile_at((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * BN + t;
      copy_code_rows<M>(slot0(k), slot0(k) + 128 * C::CODE_ROW, p.signs, row0, p.N, p.err);
    }
    int rs = 0;                 // ring slot of the next chunk and its phase
    uint32_t rph = 0;
    int cs = 0;                 // code slot of this tile's rows
    bool ok = true;
    // the two rows' norms (0 past the end), one tile ahead: B holds +-||x||
    auto norm_of = [&](int64_t row) -> uint32_t {
      return (row < p.N && JL_IN_RANGE(p.err, row, 1, p.N))
                 ? (uint32_t)__ldg(p.norms + row) & 0x7FFFu : 0u;
    };
    uint32_t n0 = norm_of(tile_at(blockIdx.x) * BN + t), n1 = norm_of(tile_at(blockIdx.x) * BN + t + 128);
    for (int64_t j = blockIdx.x; ok && j < ntiles; j += gridDim.x) {
      const int64_t nrow = tile_at(j + gridDim.x) * BN + t;
      const uint32_t nn0 = norm_of(nrow), nn1 = norm_of(nrow + 128);
      {
        const int64_t row0 = tile_at(j + (int64_t)(CODE_SLOTS - 1) * gridDim.x) * BN + t;
        const uint32_t d0 = slot0(cs == 0 ? CODE_SLOTS - 1 : cs - 1);
        copy_code_rows<M>(d0, d0 + 128 * C::CODE_ROW, p.signs, row0, p.N, p.err);
      }
      const uint32_t x0 = 0x80008000u | (n0 << 16) | n0;
      const uint32_t x1 = 0x80008000u | (n1 << 16) | n1;
      cp_async_wait<CODE_SLOTS - 1>();
      uint32_t c0w[C::CODE_WORDS], c1w[C::CODE_WORDS];
      {
        const uint32_t *s0 = reinterpret_cast<const uint32_t *>(gbase + (slot0(cs) - base));
        const uint32_t *s1 = s0 + 128 * (C::CODE_ROW / 4);
#pragma unroll
        for (int i = 0; i < C::CODE_WORDS; ++i) {
          c0w[i] = s0[i];
          c1w[i] = s1[i];
        }
      }
#pragma unroll
      for (int kc = 0; kc < C::KCH; ++kc) {
        const int s = rs;
        const uint32_t ph = rph;
        if (++rs == C::RING) {
          rs = 0;
          rph ^= 1u;
        }
        if (!wait_phase(zempty_bar(s), ph ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        uint8_t *chunk = gbase + C::OFF_Z + s * CHUNK_BYTES;
        expand_row(chunk, t, c0w[2 * kc], c0w[2 * kc + 1], x0);
        expand_row(chunk, t + 128, c1w[2 * kc], c1w[2 * kc + 1], x1);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(zfull_bar(s));
      }
      n0 = nn0;
      n1 = nn1;
      if (++cs == CODE_SLOTS) cs = 0;
    }
    cp_async_wait<0>();
  } else if (warp < MMA_WARP) {
    // ---------------- epilogue: lane = query 32 (warp % 4) + lane; half h
    // of the warps takes the 32-column groups g = h, h + 2, ...
    const int q = warp & 3;
    const int ew = warp - EXP_WARPS;
    const int h = 0;
    const int qi = 32 * q + lane;
    float *park = reinterpret_cast<float *>(gbase + C::OFF_P) + (ew * 32 + lane) * (PARK_ROWS * 33);
    // the list holds scores before the query's output scale (positive, so
    // the order is the same)
    TopList<KT> list;
    list.init();
    float published = -INFINITY;
    // insert the qualifying scores of a group held in row[32] (shared memory)
    auto insert_row = [&](const float *row, int g, int nvalid, int64_t base_row, float gb) {
      const float thr = list.thr;
      uint32_t hits = 0;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float sc = row[e];
        hits |= (32 * g + e < nvalid && sc > thr && sc >= gb) ? (1u << e) : 0u;
      }
#pragma unroll 1
      while (hits) {
        const int e = __ffs(hits) - 1;
        hits &= hits - 1;
        const float sc = row[e];
        if (sc > list.thr) list.insert(sc, (int32_t)(base_row + 32 * g + e));
      }
    };
    uint32_t tt = 0;
    for (int64_t j = blockIdx.x; j < ntiles; j += gridDim.x, ++tt) {
      const int64_t base_row = tile_at(j) * BN;
      const int nvalid = (int)((p.N - base_row) < BN ? (p.N - base_row) : BN);
      // the query's shared bound: scores below it cannot make the top KT
      const float gb = ord_float(*reinterpret_cast<volatile unsigned *>(p.gbound + qi));
      const int ab = (int)(tt % (uint32_t)C::NACC);
      if (!wait_phase(dfull_bar(ab), (tt / (uint32_t)C::NACC) & 1u, abort_flag, p.err)) break;
      __syncwarp();
      fence_after();
      const uint32_t trow =
          tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(C::D_COL + ab * BN);
      // the tile's 8 groups of 32 columns: while the accumulator is held only
      // the group maxima are taken; groups that may qualify are parked and
      // inserted once the accumulator is released (or when the rows are full)
      int np = 0;          // parked groups
      uint32_t pgs = 0;    // their group numbers, 4 bits each
      // one group: its maximum (a tree of three-input maxima, 17 steps),
      // parked if it may qualify
      auto scan_group = [&](uint32_t (&v)[32], int g) {
        float t[11];
#pragma unroll
        for (int e = 0; e < 10; ++e)
          t[e] = max3f(__uint_as_float(v[3 * e]), __uint_as_float(v[3 * e + 1]),
                       __uint_as_float(v[3 * e + 2]));
        t[10] = fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31]));
        const float gm = fmaxf(max3f(max3f(t[0], t[1], t[2]), max3f(t[3], t[4], t[5]),
                                     max3f(t[6], t[7], t[8])),
                               fmaxf(t[9], t[10]));
        if (gm > list.thr && gm >= gb) {
          float *row = park + np * 33;
#pragma unroll
          for (int e = 0; e < 32; ++e) row[e] = __uint_as_float(v[e]);
          pgs |= (uint32_t)g << (4 * np);
          ++np;
        }
      };
      auto flush = [&]() {
#pragma unroll 1
        for (int r = 0; r < np; ++r)
          insert_row(park + r * 33, (int)((pgs >> (4 * r)) & 15u), nvalid, base_row, gb);
        np = 0;
        pgs = 0;
      };
      // the tile's 8 groups of 32 columns, two at a time with the next load in
      // flight: while the accumulator is held only the group maxima are
      // taken; groups that may qualify are parked and inserted after the
      // accumulator is released (or when all rows are in use)
      uint32_t va[32], vb[32];
      ld32(trow, va);
#pragma unroll 1
      for (int g = 0; g < BN / 32; g += 2) {
        ld_wait(va);
        ld32(trow + 32 * (g + 1), vb);
        scan_group(va, g);
        ld_wait(vb);
        if (g + 2 < BN / 32) {
          ld32(trow + 32 * (g + 2), va);
        } else {  // the accumulator is read: free it
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dempty_bar(ab));
        }
        scan_group(vb, g + 1);
        // at most two groups park per pair: flush before the rows run out,
        // and after the last pair (one call site keeps the code small)
        if (np > PARK_ROWS - 2 || (g + 2 >= BN / 32 && np > 0)) flush();
      }
      // publish a better bound once the list is full
      if (list.cnt == KT && list.thr > published) {
        published = list.thr;
        atomicMax(p.gbound + qi, ord_code(published));
      }
      __syncwarp();
    }
    // this warp's list for the query (unsorted, before the output scale;
    // empty entries are -inf / -1)
    const int64_t o = (((int64_t)blockIdx.x * LISTS + h) * QM + qi) * KT;
#pragma unroll
    for (int e = 0; e < KT; ++e) {
      p.part_val[o + e] = list.val[e];
      p.part_idx[o + e] = list.idx[e];
    }
  } else {
    // ---------------- MMA issuer: the whole warp runs the loop, one elected
    // lane issues; descriptors are the base plus a 32-bit start-address add
    {
      constexpr uint32_t idesc = (1u << 4)                        // D: fp32
                                 | (0u << 7) | (0u << 10)         // A, B: fp16
                                 | ((uint32_t)(BN >> 3) << 17)    // N
                                 | ((uint32_t)(QM >> 4) << 24);   // M
      const uint64_t z0 = desc_sw128(sZ);
      const uint64_t u0 = desc_sw128(base + C::OFF_U);
      const uint32_t z_hi = (uint32_t)(z0 >> 32), z_lo0 = (uint32_t)z0;
      const uint32_t u_hi = (uint32_t)(u0 >> 32), u_lo0 = (uint32_t)u0;
      int rs = 0;
      uint32_t rph = 0;
      uint32_t tt = 0;
      bool ok = true;
      for (int64_t j = blockIdx.x; ok && j < ntiles; j += gridDim.x, ++tt) {
        // accumulator ab was read by the epilogue of tile tt - NACC
        const uint32_t ab = tt % (uint32_t)C::NACC;
        if (!__all_sync(0xffffffffu, wait_phase(dempty_bar((int)ab),
                                                ((tt / (uint32_t)C::NACC) & 1u) ^ 1u,
                                                abort_flag, p.err)))
          break;
        fence_after();
        const uint32_t dt = tmem_base + (uint32_t)C::D_COL + ab * (uint32_t)BN;
        for (int kc = 0; kc < C::KCH; ++kc) {
          const int s = rs;
          const uint32_t ph = rph;
          if (++rs == C::RING) {
            rs = 0;
            rph ^= 1u;
          }
          if (!__all_sync(0xffffffffu, wait_phase(zfull_bar(s), ph, abort_flag, p.err))) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t zlo = z_lo0 + (uint32_t)s * (uint32_t)(CHUNK_BYTES >> 4);
          const uint32_t ulo = u_lo0 + (uint32_t)kc * (uint32_t)(C::U_CHUNK >> 4);
          uint32_t el;
          asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.u32 %0, 1, 0, e;\n}\n"
                       : "=r"(el));
          if (el) {
#pragma unroll
            for (int kk = 0; kk < CHUNK_K / 16; ++kk) {
              const uint64_t bdesc = ((uint64_t)z_hi << 32) | (uint64_t)(zlo + (uint32_t)(kk * 2));
              const uint32_t acc = (kc > 0 || kk > 0) ? 1u : 0u;
              if constexpr (C::U_SMEM)
                mma_ss(dt, ((uint64_t)u_hi << 32) | (uint64_t)(ulo + (uint32_t)(kk * 2)),
                           bdesc, idesc, acc);
              else
                mma_ts(dt, tmem_base + (uint32_t)(kc * 32 + kk * 8), bdesc, idesc, acc);
            }
            commit(zempty_bar(s));
          }
          __syncwarp();
        }
        if (!ok) break;
        uint32_t el2;
        asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.u32 %0, 1, 0, e;\n}\n"
                     : "=r"(el2));
        if (el2) commit(dfull_bar((int)ab));
        __syncwarp();
      }
      if (tt > 0 && ok && lane == 0) {  // the last tile's MMAs complete before TMEM is freed
        const unsigned long long t0 = globaltimer();
        const int lb = (int)((tt - 1) % C::NACC);
        while (!mbar_try_wait(dfull_bar(lb), ((tt - 1) / (uint32_t)C::NACC) & 1u) &&
               globaltimer() - t0 < WAIT_LIMIT_NS) {
        }
      }
      __syncwarp();
    }
  }

  fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem_base),
                 "n"(TMEM_COLS)
                 : "memory");
  }
}

// --------------------------------------------------------------------------
// Merge: per query, the k best of all CTAs' lists, best first (ties to the
// lower index); entries beyond the candidates are (-1, -inf).  Output mode
// writes them (scores times the query's output scale); bound mode writes the
// k-th best as the query's shared bound (none if fewer than k candidates).
__device__ __forceinline__ bool better(float a, int32_t ia, float b, int32_t ib) {
  return a > b || (a == b && (unsigned)ia < (unsigned)ib);
}

// The best (value, index, position) of a warp: each lane offers its own best
// (position < 0 = none), the winner is broadcast to all lanes.
__device__ __forceinline__ void warp_best(float &bv, int32_t &bi, int &bp) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
    const int op = __shfl_xor_sync(0xffffffffu, bp, o);
    if (op >= 0 && (bp < 0 || better(ov, oi, bv, bi))) {
      bv = ov;
      bi = oi;
      bp = op;
    }
  }
}

// Two levels: each warp takes the k best of its slice of the candidates
// (lane l owns slice entries l, l + 32, ...; the winning lane strikes its own
// entry, so a round needs no block barrier), then warp 0 takes the k best of
// the warps' lists.
__global__ void __launch_bounds__(MERGE_THREADS) search_merge_kernel(
    const float *__restrict__ part_val, const int32_t *__restrict__ part_idx, int ctas, int kt,
    int k, const float *__restrict__ qscale, int32_t *__restrict__ out_idx,
    float *__restrict__ out_scores, unsigned *__restrict__ bound_out) {
  constexpr int NW = MERGE_THREADS / 32;
  extern __shared__ uint8_t mg_smem[];
  const int ncand = ctas * LISTS * kt;
  float *cv = reinterpret_cast<float *>(mg_smem);
  int32_t *ci = reinterpret_cast<int32_t *>(cv + ncand);
  __shared__ float wv[NW * 16];
  __shared__ int32_t wi[NW * 16];
  const int qi = blockIdx.x;
  for (int e = threadIdx.x; e < ncand; e += MERGE_THREADS) {
    const int list = e / kt, j = e - list * kt;  // list = cta * LISTS + half
    const int64_t o = ((int64_t)list * QM + qi) * kt + j;
    cv[e] = part_val[o];
    ci[e] = part_idx[o];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int per = (ncand + NW - 1) / NW;
  const int e0 = w * per, e1 = min(ncand, e0 + per);
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int32_t bi = -1;
    int bp = -1;
    for (int e = e0 + lane; e < e1; e += 32)
      if (ci[e] >= 0 && (bp < 0 || better(cv[e], ci[e], bv, bi))) {
        bv = cv[e];
        bi = ci[e];
        bp = e;
      }
    const int mine = bp;
    warp_best(bv, bi, bp);
    if (bp >= 0 && bp == mine) ci[bp] = -1;  // the owner strikes the winner
    if (lane == 0) {
      wv[w * 16 + r] = bv;
      wi[w * 16 + r] = bp >= 0 ? bi : -1;
    }
    __syncwarp();
  }
  __syncthreads();
  if (w != 0) return;
  // warp 0: NW lists of k, lane l owns entries l, l + 32, ... of the NW x 16 grid
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int32_t bi = -1;
    int bp = -1;
    for (int e = lane; e < NW * 16; e += 32)
      if ((e & 15) < k && wi[e] >= 0 && (bp < 0 || better(wv[e], wi[e], bv, bi))) {
        bv = wv[e];
        bi = wi[e];
        bp = e;
      }
    const int mine = bp;
    warp_best(bv, bi, bp);
    if (bp >= 0 && bp == mine) wi[bp] = -1;
    if (lane == 0) {
      if (bound_out) {
        if (r == k - 1) bound_out[qi] = bp >= 0 ? ord_code(bv) : 0u;
      } else {
        out_idx[(int64_t)qi * k + r] = bp >= 0 ? bi : -1;
        out_scores[(int64_t)qi * k + r] = bp >= 0 ? bv * qscale[qi] : -INFINITY;
      }
    }
    __syncwarp();
  }
}

// list length per query and CTA (k <= JL_SEARCH_MAX_K = 16): a longer list
// would not fit the epilogue's registers
static int list_len(int) { return 16; }

template <int M, int KT>
static cudaError_t launch_pass(const Params &p, int grid, cudaStream_t stream) {
  using C = Cfg<M>;
  cudaError_t e = cudaFuncSetAttribute(search_tc_kernel<M, KT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  search_tc_kernel<M, KT><<<grid, THREADS, C::SMEM, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace srch

size_t search_workspace_bytes(int nq, int m, int k) {
  (void)nq;
  const size_t u = (size_t)srch::QM * m * sizeof(float);
  const size_t lists = (size_t)srch::MAX_CTAS * srch::LISTS * srch::QM * srch::list_len(k);
  return (u + 255) / 256 * 256 + lists * (sizeof(float) + sizeof(int32_t)) +
         srch::QM * (sizeof(unsigned) + sizeof(float)) + 256;
}

cudaError_t launch_search(const void *Q, bool q_f32, int nq, const uint16_t *S, int m, int d,
                          const uint32_t *signs, const uint16_t *norms, int64_t N, int k,
                          int32_t *out_idx, float *out_scores, void *workspace,
                          cudaStream_t stream) {
  using namespace srch;
  int *err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  const int kt = list_len(k);
  uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
  float *U = reinterpret_cast<float *>(ws);
  const size_t u_bytes = ((size_t)QM * m * sizeof(float) + 255) / 256 * 256;
  float *part_val = reinterpret_cast<float *>(ws + u_bytes);
  int32_t *part_idx = reinterpret_cast<int32_t *>(part_val + (size_t)MAX_CTAS * LISTS * QM * kt);
  unsigned *gbound = reinterpret_cast<unsigned *>(part_idx + (size_t)MAX_CTAS * LISTS * QM * kt);
  float *qscale = reinterpret_cast<float *>(gbound + QM);
  const int64_t num_tiles = (N + BN - 1) / BN;
  int64_t grid64 = device_sm_count();
  if (grid64 > MAX_CTAS) grid64 = MAX_CTAS;
  if (grid64 > num_tiles) grid64 = num_tiles;
  const int grid = (int)grid64;
  const size_t qbytes = (size_t)d * (q_f32 ? 4 : 2);
  const size_t msmem = (size_t)grid * LISTS * kt * (sizeof(float) + sizeof(int32_t));
  cudaError_t e = cudaFuncSetAttribute(search_merge_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
  if (e != cudaSuccess) return e;
  for (int q0 = 0; q0 < nq; q0 += QM) {
    const int nqp = nq - q0 < QM ? nq - q0 : QM;
    e = launch_query_projection(reinterpret_cast<const uint8_t *>(Q) + (size_t)q0 * qbytes,
                                q_f32, S, U, nqp, m, d, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(gbound, 0, QM * sizeof(unsigned), stream);  // no bound yet
    if (e != cudaSuccess) return e;
    Params p{signs, norms, U, part_val, part_idx, gbound, qscale, N, num_tiles, 0, 1, nqp,
             (float)(1.2533141373155002512 / (double)m), err};
    auto run = [&](const Params &pp) -> cudaError_t {
#define JL_CASE(MM) \
      if (m == MM) return launch_pass<MM, 16>(pp, grid, stream);
      JL_CASE(64) JL_CASE(128) JL_CASE(256) JL_CASE(512)
#undef JL_CASE
      return cudaErrorNotSupported;
    };
    // warm start: about 4 tiles per CTA spread over the index, merged into
    // each query's starting bound (the 16th best of the sample)
    const int64_t sample_step = num_tiles / ((int64_t)grid * 4);
    if (sample_step >= 2) {
      Params ps = p;
      ps.tile_step = sample_step;
      ps.num_tiles = (num_tiles + sample_step - 1) / sample_step;
      e = run(ps);
      if (e != cudaSuccess) return e;
      search_merge_kernel<<<nqp, MERGE_THREADS, msmem, stream>>>(
          part_val, part_idx, grid, kt, kt, qscale, nullptr, nullptr, gbound);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    e = run(p);
    if (e != cudaSuccess) return e;
    search_merge_kernel<<<nqp, MERGE_THREADS, msmem, stream>>>(
        part_val, part_idx, grid, kt, k, qscale, out_idx + (size_t)q0 * k,
        out_scores + (size_t)q0 * k, nullptr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace jlk
