// dequant_tc.cu -- explicit dequantizers on the 5th-generation tensor cores.
//
// QJL codes: the dequantizer Q^-1(z) = sqrt(pi/2)/d * S^T z of "The Geometry
// of Forgetting: How Three Papers Cracked KV Cache Quantization", section
// "QJL: one bit, zero parameters, unbiased inner products", taken with m
// sketch rows and with the stored norm restoring the magnitude (same page,
// "PolarQuant" section):
//     khat = sqrt(pi/2)/m * ||k|| * S^T z,   z_i = +1 if code bit i is set.
// The reconstruction error E||k - khat||^2 is the page's D_mse for this
// quantizer.
//
// TurboQuant-prod codes (same page, "TurboQuant: bridging MSE and inner
// product, in two stages": the QJL estimate of the residual is added back to
// the stage-one reconstruction), in the rotated frame, mapped back with the
// inverse of the stored rotation and scaled by the key norm:
//     khat = ||k|| * Pi^{-1} ( c[cell] + sqrt(pi/2)/m * ||r|| * S^T z )
//          = ||k|| * R a,   R = [Pi^{-1} | Pi^{-1} S^T]  (d x (d + m)),
//     a = [c[cell_0 .. cell_{d-1}] ; alpha z],  alpha = sqrt(pi/2)/m * ||r||.
// R is built once (turbo_basis_kernel); a holds binary16 centroids and
// +-alpha, so a key costs one fp16 contraction of length d + m.
//
// For a tile of 128 codes, Khat = A B is a dense contraction (M = 128 codes,
// N = d, K = m or d + m): tcgen05.mma with A read from tensor memory, B from
// shared memory (128-byte swizzle, K-major) and the fp32 accumulator in
// tensor memory.
//   * A is expanded from the code bits by threads straight into tensor
//     memory, one K-chunk of 64 coordinates (32 columns of 16-bit pairs, one
//     tcgen05.st per thread) at a time, into a ring of chunks; it never
//     passes through shared memory.  A pair holds coordinates (p, p + 16) of
//     a 32-bit code word.  QJL: bf16 +-1 with one shift and one LOP3,
//     ((w << (15 - p)) & 0x80008000) ^ 0xBF80BF80.  TurboQuant: the cell's
//     centroid as binary16, its magnitude chosen by the XNOR of each lower
//     plane with the top plane (the codebook is odd-symmetric) and its sign
//     by the top plane; then the residual signs as +-alpha.
//   * B (S^T, or R^T for TurboQuant) stays resident; its K order is the same
//     permutation of each 32-coordinate block, so the contraction is
//     unchanged.  TurboQuant interleaves its K-chunks (centroid chunk i at
//     2 i, sign chunk i at 2 i + 1); at d = 128 each expander part thus
//     expands one chunk of each kind.
//   * The epilogue scales row r by sqrt(pi/2)/m * ||k_r|| (QJL) or ||k_r||
//     (TurboQuant), rounds to bf16, writes its 32 rows into a
//     128-byte-swizzled staging tile in shared memory and stores them with
//     bulk-tensor copies (which also clip rows past the last code).
//   * An expander thread copies its part of its code row of the tile two
//     ahead into a shared-memory ring with cp.async while it expands the
//     current one.
//
// One persistent CTA per SM, 13 warps with fixed roles:
//   warps 0-7  expand: warp w writes TMEM lane quadrant w % 4 (code rows
//              32 (w % 4) .. + 31 of the tile) for part w / 4 of the tile's
//              K-chunks (the first or the second half), so two warps expand
//              each row at once; each thread copies its part of its code
//              row two tiles ahead.
//   warps 8-11 epilogue: warp w reads TMEM lane quadrant w % 4.
//   warp 12    owns the TMEM allocation; one elected lane issues the MMAs of a tile
//              into one of two accumulators and commits them to the barriers
//              that free the A chunks and publish the accumulator.
// Every mbarrier wait is bounded (about 2 s of GPU time); a wait that runs
// out records DERR_TC_WAIT_TIMEOUT, raises a shared abort flag, and the CTA
// still frees its TMEM.
#include "jl_common.cuh"
#include "jl_internal.h"
#include "jl_tc.cuh"

#include <cuda_fp16.h>
#include <cudaTypedefs.h>

namespace jlk {

using namespace tcx;
namespace dq {

constexpr int BM = 128;          // codes per tile (MMA M)
constexpr int CHUNK_K = 64;      // coordinates per A chunk
constexpr int CHUNK_COLS = CHUNK_K / 2;  // TMEM columns of an A chunk (16-bit pairs)
constexpr int EXP_PARTS = 2;     // expander warps per TMEM lane quadrant
constexpr int EXP_WARPS = 4 * EXP_PARTS, EPI_WARPS = 4;
constexpr int MMA_WARP = EXP_WARPS + EPI_WARPS;
constexpr int THREADS = (MMA_WARP + 1) * 32;
constexpr int CODE_SLOTS = 3;    // code rows in flight: the tile and two ahead
constexpr uint32_t SIGN2 = 0x80008000u;  // sign bits of a 16-bit pair

// TB = 0: QJL codes (m/32 sign words, one binary16 norm per key).
// TB = 1..3: TurboQuant-prod codes (TB cell planes of d bits, then m sign
// bits; a binary16 (||k||, ||r||) pair per key); d = m = 64 or 128.
template <int M, int D, int TB>
struct Cfg {
  static constexpr bool TURBO = TB > 0;
  static constexpr int K = TURBO ? D + M : M;         // contraction length
  static constexpr int KCH = K / CHUNK_K;             // A chunks per tile (>= 1)
  static constexpr int B_CHUNK = D * 128;             // one K-chunk of B
  static constexpr int B_BYTES = K * D * 2;
  // output staging: per epilogue warp, 32 rows x d bf16 as D/64 swizzled
  // boxes of 32 x 128 B, two buffers per warp
  static constexpr int OBOX = 32 * 128;
  static constexpr int OWARP = (D / 64) * OBOX;
  static constexpr int KP = (KCH + EXP_PARTS - 1) / EXP_PARTS;  // chunks per part
  // code bytes of one part of a row in the ring: QJL, the part's 2 words per
  // chunk; TurboQuant, 8 bytes of every cell plane and of the sign words,
  // then the norm pair (padded to 8)
  static constexpr int PART_BYTES = TURBO ? 8 * (TB + 1) + 8 : KP * 8;
  static constexpr int CODE_ROW = TURBO ? EXP_PARTS * PART_BYTES : M / 8;
  static constexpr int CODE_BYTES_G = TURBO ? (TB * D + M) / 8 : M / 8;  // per key in HBM
  static constexpr int C_BYTES = CODE_SLOTS * BM * CODE_ROW;
  static constexpr int OBUF = 2;
  static constexpr int O_BYTES = EPI_WARPS * OBUF * OWARP;
  // tensor memory: accumulators at columns [0, 2d), A chunks after them
  static constexpr int ACC = 2;
  static constexpr int TMEM_COLS = 512;
  static constexpr int A_COL0 = ACC * D;
  static constexpr int RING_RAW = (TMEM_COLS - A_COL0) / CHUNK_COLS;
  static constexpr int RING = RING_RAW > 8 ? 8 : RING_RAW;
  static constexpr int OFF_O = B_BYTES;
  static constexpr int OFF_C = OFF_O + O_BYTES;
  static constexpr int OFF_BAR = OFF_C + C_BYTES;
  static constexpr int NBAR = 2 * RING + 2 * ACC;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + align slack
  static_assert(K % CHUNK_K == 0 && RING >= 2, "A ring");
  static_assert(A_COL0 + RING * CHUNK_COLS <= TMEM_COLS, "tensor memory columns");
  static_assert(!TURBO || ((D == 128 || D == 64) && M == D && TB <= 3), "TurboQuant shapes");
  static_assert(!TURBO || KCH % EXP_PARTS == 0, "whole chunks per part");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct Params {
  const uint32_t *codes;  // n x code words
  const uint16_t *norms;  // n binary16 (QJL) or n x 2 (TurboQuant)
  const uint16_t *B;      // QJL: S, m x d bf16; TurboQuant: R, d x (d + m) binary16
  int64_t n, num_tiles;
  float coef;             // sqrt(pi/2) / m
  uint32_t mag[4];        // TurboQuant: centroid magnitudes a_0 < .. (binary16 pairs)
  uint32_t dmag01, dmag23;  // a_0 ^ a_1, a_2 ^ a_3 (binary16 bits)
  int *err;
};


// 4-byte async copy global -> shared; src_bytes < 4 zero-fills.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src,
                                           int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst),
               "l"(src), "r"(src_bytes)
               : "memory");
}

// Bulk-tensor store of a staged box (shared -> global, never multicast) and
// the waits on this thread's outstanding stores.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];\n" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
}
// all but the newest N groups have finished reading shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;\n" ::"n"(N) : "memory");
}
// every store has completed
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
}


// Position of coordinate i of a 32-coordinate block in the operand's K
// order: 16-bit pair j holds coordinates j (low half) and j + 16 (high half).
__host__ __device__ __forceinline__ int k_slot(int i) {
  const int j = i & 15, h = (i >> 4) & 1;
  return (i & ~31) + 2 * j + h;
}

// Byte offset of element (row r, K position k) in a K-major, 128-byte-swizzle
// operand of `rows` rows: 64-element K-chunks of rows x 128 B, 16-byte units
// of a row permuted by (row & 7).
__device__ __forceinline__ uint32_t sw128_offset(int r, int k, int rows) {
  const int kc = k >> 6, kin = k & 63;
  return (uint32_t)(kc * rows * 128 + r * 128 + ((((kin >> 3) ^ (r & 7)) << 4)) + (kin & 7) * 2);
}

// TurboQuant centroid pairs of one code word per plane: pair j holds the
// binary16 centroids of coordinates j and j + 16 of the 32 the words cover.
// The cell's top plane bit gives the sign (set: positive); each lower plane
// bit XNOR the top one gives a bit of the magnitude's index (the codebook is
// c[H + i] = a_i, c[H - 1 - i] = -a_i).
template <int TB>
__device__ __forceinline__ void centroid_pairs(const uint32_t (&w)[TB], const Params &p,
                                               uint32_t *z) {
  if constexpr (TB == 1) {
    const uint32_t k = SIGN2 | p.mag[0];
#pragma unroll
    for (int j = 0; j < 16; ++j) z[j] = ((w[0] << (15 - j)) & SIGN2) ^ k;
  } else if constexpr (TB == 2) {
    const uint32_t x = ~(w[0] ^ w[1]);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t mag = p.mag[0] ^ (((x >> j) & 0x00010001u) * p.dmag01);
      z[j] = mag ^ (((w[1] << (15 - j)) & SIGN2) ^ SIGN2);
    }
  } else {
    const uint32_t x0 = ~(w[0] ^ w[2]), x1 = ~(w[1] ^ w[2]);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t u0 = (x0 >> j) & 0x00010001u;
      const uint32_t lo = p.mag[0] ^ (u0 * p.dmag01);
      const uint32_t hi = p.mag[2] ^ (u0 * p.dmag23);
      const uint32_t sel = ((x1 >> j) & 0x00010001u) * 0xFFFFu;
      const uint32_t mag = (hi & sel) | (lo & ~sel);
      z[j] = mag ^ (((w[2] << (15 - j)) & SIGN2) ^ SIGN2);
    }
  }
}

template <int M, int D, int TB>
__global__ void __launch_bounds__(THREADS, 1)
    dequant_tc_kernel(const __grid_constant__ CUtensorMap tmap_out, const Params p) {
  using C = Cfg<M, D, TB>;
  extern __shared__ uint8_t dq_smem_raw[];
  const uint32_t raw = smem_u32(dq_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = dq_smem_raw + (base - raw);
  const uint32_t sB = base;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto afull_bar = [&](int s) { return bar0 + 8u * s; };               // A chunk written
  auto aempty_bar = [&](int s) { return bar0 + 8u * (C::RING + s); };  // A chunk consumed
  auto accfull_bar = [&](int a) { return bar0 + 8u * (2 * C::RING + a); };
  auto accempty_bar = [&](int a) { return bar0 + 8u * (2 * C::RING + C::ACC + a); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int *abort_flag =
      reinterpret_cast<volatile int *>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::RING; ++s) {
      mbar_init(afull_bar(s), 4);            // one arrive per quadrant's expander warp
      mbar_init(aempty_bar(s), 1);           // MMA commit
    }
    for (int a = 0; a < C::ACC; ++a) {
      mbar_init(accfull_bar(a), 1);          // MMA commit
      mbar_init(accempty_bar(a), EPI_WARPS); // epilogue warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
        "tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::"r"(
            smem_u32(tmem_holder)),
        "n"(C::TMEM_COLS)
        : "memory");
  }
  // B into shared memory, once: 16-byte unit (row n, K positions 8u..8u+7)
  // per thread and step; K position k of a chunk holds coordinate i with
  // k_slot(i) = k
  if constexpr (!C::TURBO) {
    for (int e = threadIdx.x; e < D * (M / 8); e += THREADS) {
      const int n = e % D, u = e / D;
      uint32_t pk[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint16_t h2[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int k = 8 * u + 2 * q + hh;           // K position
          const int blk = k & ~31, jj = (k & 31) >> 1, h = k & 1;
          const int i = blk + jj + 16 * h;            // coordinate at k
          h2[hh] = __ldg(p.B + (int64_t)i * D + n);   // S[i][n]
        }
        pk[q] = (uint32_t)h2[0] | ((uint32_t)h2[1] << 16);
      }
      *reinterpret_cast<uint4 *>(gbase + sw128_offset(n, 8 * u, D)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  } else {
    // R row n is K-contiguous: the unit's low halves are 4 consecutive
    // columns, its high halves the 4 columns 16 later
    for (int e = threadIdx.x; e < D * (C::K / 8); e += THREADS) {
      const int n = e % D, ug = e / D;
      const int kc = ug >> 3, u = ug & 7;
      const int col0 = ((kc & 1) ? D + 64 * (kc >> 1) : 64 * (kc >> 1)) + 32 * (u >> 2) +
                       4 * (u & 3);
      const int64_t off = (int64_t)n * (D + M) + col0;
      uint2 lo = make_uint2(0u, 0u), hi = make_uint2(0u, 0u);
      if (JL_IN_RANGE(p.err, off, 20, (int64_t)D * (D + M))) {
        lo = __ldg(reinterpret_cast<const uint2 *>(p.B + off));
        hi = __ldg(reinterpret_cast<const uint2 *>(p.B + off + 16));
      }
      *reinterpret_cast<uint4 *>(gbase + sw128_offset(n, 8 * ug, D)) =
          make_uint4(__byte_perm(lo.x, hi.x, 0x5410), __byte_perm(lo.x, hi.x, 0x7632),
                     __byte_perm(lo.y, hi.y, 0x5410), __byte_perm(lo.y, hi.y, 0x7632));
    }
  }
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int64_t ntiles = p.num_tiles;

  if (warp < EXP_WARPS) {
    // ---------------- expand: quadrant q = warp % 4 (row r = 32 q + lane),
    // part pt = warp / 4: chunks [kc0, kc0 + nk) of every tile; the part's
    // code words of the tile two ahead are copied meanwhile
    const int q = warp & 3, pt = warp >> 2;
    const int r = 32 * q + lane;
    constexpr int KP = C::KP;
    const int kc0 = pt * KP;
    const int nk = C::KCH - kc0 < KP ? C::KCH - kc0 : KP;
    bool ok = nk > 0;
    const uint32_t crow =
        base + C::OFF_C + r * C::CODE_ROW + pt * (C::TURBO ? C::PART_BYTES : KP * 8);
    auto code_slot = [&](int slot) { return crow + (uint32_t)(slot * BM * C::CODE_ROW); };
    auto copy_part = [&](uint32_t dst, int64_t row) {
      if constexpr (!C::TURBO) {
        const bool live = row < p.n && JL_IN_RANGE(p.err, row * (M / 8) + pt * KP * 8, KP * 8,
                                                   p.n * (M / 8));
        const uint8_t *src =
            reinterpret_cast<const uint8_t *>(p.codes + (live ? row : 0) * (M / 32)) + pt * KP * 8;
        if constexpr (KP * 8 >= 16) {
#pragma unroll
          for (int u = 0; u < KP * 8 / 16; ++u) cp_async_16(dst + 16 * u, src + 16 * u, live ? 16 : 0);
        } else {
          cp_async_8(dst, src, live ? 8 : 0);
        }
      } else {
        // 8 bytes (the 64 coordinates of the part's chunk index kc0 / 2) of
        // each cell plane and of the sign words, then the norm pair
        const bool live = row < p.n &&
                          JL_IN_RANGE(p.err, row * C::CODE_BYTES_G, C::CODE_BYTES_G,
                                      p.n * C::CODE_BYTES_G) &&
                          JL_IN_RANGE(p.err, 2 * row, 2, 2 * p.n);
        const int64_t rr = live ? row : 0;
        const uint8_t *src =
            reinterpret_cast<const uint8_t *>(p.codes) + rr * C::CODE_BYTES_G + 8 * (kc0 >> 1);
#pragma unroll
        for (int pl = 0; pl <= TB; ++pl) cp_async_8(dst + 8 * pl, src + pl * (D / 8), live ? 8 : 0);
        cp_async_4(dst + 8 * (TB + 1), p.norms + 2 * rr, live ? 4 : 0);
      }
      cp_async_commit();
    };
    if (ok)
      for (int k = 0; k < CODE_SLOTS - 1; ++k)
        copy_part(code_slot(k), ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * BM + r);
    int cs = 0;                    // code slot of this tile's words
    // ring slot and phase of this part's first chunk of the tile: global
    // chunk it * KCH + kc0, advanced by KCH per tile without a division
    int rs0 = kc0 % C::RING;
    uint32_t rph0 = (uint32_t)((kc0 / C::RING) & 1);
    constexpr int NW = C::TURBO ? 2 * TB + 3 : 2 * KP;  // words of a part's slot
    for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      copy_part(code_slot(cs == 0 ? CODE_SLOTS - 1 : cs - 1),
                (tile + (int64_t)(CODE_SLOTS - 1) * gridDim.x) * BM + r);
      cp_async_wait<CODE_SLOTS - 1>();  // this tile's words have landed
      uint32_t cur[NW];
      {
        const uint8_t *src = gbase + (code_slot(cs) - base);
#pragma unroll
        for (int i = 0; i < NW; ++i) cur[i] = reinterpret_cast<const uint32_t *>(src)[i];
      }
      // TurboQuant: +-alpha pairs for the sign chunk, alpha = sqrt(pi/2)/m ||r||
      // rounded to binary16 (rows past the end have a zero norm pair)
      uint32_t kalpha = 0;
      if constexpr (C::TURBO) {
        const float alpha =
            p.coef * __half2float(__ushort_as_half((uint16_t)(cur[2 * TB + 2] >> 16)));
        const uint32_t a16 = (uint32_t)__half_as_ushort(__float2half_rn(alpha));
        kalpha = SIGN2 | (a16 << 16) | a16;
      }
      int s = rs0;
      uint32_t ph = rph0;
#pragma unroll
      for (int kk = 0; kk < KP; ++kk) {
        if (kk >= nk) break;
        if (kk > 0 && ++s == C::RING) {  // global chunk it * KCH + kc0 + kk
          s = 0;
          ph ^= 1u;
        }
        if (!wait_phase(aempty_bar(s), ph ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        // the chunk's 32 TMEM columns of row r: column 16 h + j holds the
        // pair (j, j + 16) of the chunk's code word h
        uint32_t z[32];
        if constexpr (!C::TURBO) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t w = cur[2 * kk + half];  // rows past the end expand a zero code
#pragma unroll
            for (int j = 0; j < 16; ++j)
              z[16 * half + j] = ((w << (15 - j)) & SIGN2) ^ 0xBF80BF80u;
          }
        } else if (((kc0 + kk) & 1) == 0) {         // centroid chunk (kc0 + kk) / 2
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t w[TB];
#pragma unroll
            for (int pl = 0; pl < TB; ++pl) w[pl] = cur[2 * pl + half];
            centroid_pairs<TB>(w, p, z + 16 * half);
          }
        } else {                                    // sign chunk (kc0 + kk) / 2
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t w = cur[2 * TB + half];
#pragma unroll
            for (int j = 0; j < 16; ++j) z[16 * half + j] = ((w << (15 - j)) & SIGN2) ^ kalpha;
          }
        }
        st32(tmem_base + ((uint32_t)(32 * q) << 16) +
                      (uint32_t)(C::A_COL0 + s * CHUNK_COLS), z);
        st_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull_bar(s));
      }
      // next tile: its first chunk of this part is KCH chunks later
      rs0 += C::KCH;
      while (rs0 >= C::RING) {
        rs0 -= C::RING;
        rph0 ^= 1u;
      }
      if (++cs == CODE_SLOTS) cs = 0;
    }
    cp_async_wait<0>();  // no copy outlives the CTA
  } else if (warp < MMA_WARP) {
    // ---------------- epilogue: TMEM lane quadrant warp % 4; rows are staged
    // in shared memory (128-byte swizzle) and written by bulk-tensor stores
    const int q = warp & 3;
    const int ew = warp - EXP_WARPS;
    // the row's stored norm (||k||), 0 past the end; loaded a tile ahead, so
    // that its latency hides behind the current tile rather than stalling
    // the warp once the accumulator is ready
    constexpr int NSTRIDE = C::TURBO ? 2 : 1;  // binary16s per key
    auto load_norm = [&](int64_t tl) -> uint16_t {
      const int64_t row = tl * BM + 32 * q + lane;
      uint16_t h = 0;
      if (tl < ntiles && row < p.n && JL_IN_RANGE(p.err, NSTRIDE * row, 1, NSTRIDE * p.n))
        h = __ldg(p.norms + NSTRIDE * row);
      return h;
    };
    uint16_t nrm_next = load_norm(blockIdx.x);
    int64_t t = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++t) {
      const int a = (int)(t & 1);
      const uint32_t aph = (uint32_t)((t >> 1) & 1);
      const uint16_t nrm = nrm_next;
      nrm_next = load_norm(tile + gridDim.x);
      const float f = (C::TURBO ? 1.f : p.coef) * __half2float(__ushort_as_half(nrm));
      const int ob = (int)(t % C::OBUF);
      uint8_t *stage = gbase + C::OFF_O + (ew * C::OBUF + ob) * C::OWARP;
      // the staging buffer's previous stores must have read it
      if (lane == 0) bulk_wait_read<C::OBUF - 1>();
      __syncwarp();
      if (!wait_phase(accfull_bar(a), aph, abort_flag, p.err)) break;
      __syncwarp();
      fence_after();
      const uint32_t trow = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * D);
      // 32 columns: scale, round to bf16, stage as 4 units of 16 B in box
      // c0/64, row `lane`
      auto emit = [&](const uint32_t (&v)[32], int c0) {
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          o[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * f, __uint_as_float(v[2 * e + 1]) * f);
        uint8_t *box = stage + (c0 >> 6) * C::OBOX + lane * 128;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int unit = ((c0 & 63) >> 3) + e;
          *reinterpret_cast<uint4 *>(box + ((unit ^ (lane & 7)) << 4)) =
              make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
      };
      // the loads are double-buffered: group g + 1 is in flight while g is
      // emitted
      uint32_t va[32], vb[32];
      ld32(trow, va);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 64) {
        ld_wait(va);
        ld32(trow + c0 + 32, vb);
        emit(va, c0);
        ld_wait(vb);
        if (c0 + 64 < D) ld32(trow + c0 + 64, va);
        emit(vb, c0 + 32);
      }
      fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(accempty_bar(a));
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_store_2d(&tmap_out, smem_u32(stage + bx * C::OBOX), bx * 64,
                       (int)(tile * BM + 32 * q));
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();  // stores complete before the CTA exits
    __syncwarp();
  } else {
    // ---------------- MMA issuer: the whole warp runs the loop, one elected
    // lane issues; the B descriptor is the base plus a 32-bit start-address add
    {
      constexpr uint32_t idesc = idesc_f16(BM, D, C::TURBO ? 0 : 1);  // fp16 or bf16
      const uint64_t b0 = desc_sw128(sB);
      const uint32_t b_hi = (uint32_t)(b0 >> 32), b_lo0 = (uint32_t)b0;
      int rs = 0;
      uint32_t rph = 0;
      uint32_t t = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++t) {
        const int a = (int)(t & 1u);
        const uint32_t aph = (t >> 1) & 1u;
        if (!__all_sync(0xffffffffu, wait_phase(accempty_bar(a), aph ^ 1u, abort_flag, p.err)))
          break;
        fence_after();
        for (int kc = 0; kc < C::KCH; ++kc) {
          const int s = rs;
          const uint32_t ph = rph;
          if (++rs == C::RING) {
            rs = 0;
            rph ^= 1u;
          }
          if (!__all_sync(0xffffffffu, wait_phase(afull_bar(s), ph, abort_flag, p.err))) {
            ok = false;
            break;
          }
          fence_after();
          if (elect_one()) {
            const uint32_t blo = b_lo0 + (uint32_t)kc * (uint32_t)(C::B_CHUNK >> 4);
#pragma unroll
            for (int kk = 0; kk < CHUNK_K / 16; ++kk) {  // K = 16: 8 columns of A
              const uint32_t atm = tmem_base + (uint32_t)(C::A_COL0 + s * CHUNK_COLS + kk * 8);
              const uint64_t bdesc = ((uint64_t)b_hi << 32) | (uint64_t)(blo + (uint32_t)(kk * 2));
              mma_ts(tmem_base + a * D, atm, bdesc, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
            }
            commit(aempty_bar(s));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) commit(accfull_bar(a));
        __syncwarp();
      }
      // drain: the last accumulator's MMAs must be complete before TMEM is freed
      if (t > 0 && ok && lane == 0) {
        const uint32_t tl = t - 1;
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(accfull_bar((int)(tl & 1u)), (tl >> 1) & 1u) &&
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
                 "n"(C::TMEM_COLS)
                 : "memory");
  }
}

// out [n][d] bf16, boxes of 64 columns (128 B) x 32 rows, 128-byte swizzle
static bool make_out_map(CUtensorMap *map, uint16_t *out, int64_t n, int d) {
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)n};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int M, int D, int TB>
cudaError_t launch_t(Params p, uint16_t *out, cudaStream_t stream) {
  using C = Cfg<M, D, TB>;
  p.err = device_error_ptr();
  if (!p.err) return cudaErrorInvalidSymbol;
  CUtensorMap tmap;
  if (!make_out_map(&tmap, out, p.n, D)) return cudaErrorInvalidValue;
  p.num_tiles = (p.n + BM - 1) / BM;
  p.coef = (float)(1.2533141373155002512 / (double)M);
  cudaError_t e = cudaFuncSetAttribute(dequant_tc_kernel<M, D, TB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t sms = device_sm_count();
  const int64_t grid = p.num_tiles < sms ? p.num_tiles : sms;
  dequant_tc_kernel<M, D, TB><<<(int)grid, THREADS, C::SMEM, stream>>>(tmap, p);
  return cudaGetLastError();
}

// R = [Pinv | Pinv S^T] rounded to binary16: one thread per element, the
// products accumulated in fp32
constexpr int BASIS_THREADS = 256;
__global__ void __launch_bounds__(BASIS_THREADS)
    turbo_basis_kernel(const float *__restrict__ Pinv, const uint16_t *__restrict__ S, int m,
                       int d, uint16_t *__restrict__ basis, int *err) {
  const int idx = blockIdx.x * BASIS_THREADS + threadIdx.x;
  const int cols = d + m;
  if (idx >= d * cols) return;
  const int j = idx / cols, c = idx % cols;
  float v = 0.f;
  if (c < d) {
    if (JL_IN_RANGE(err, j * d + c, 1, d * d)) v = Pinv[j * d + c];
  } else {
    const int l = c - d;
    if (JL_IN_RANGE(err, j * d, d, d * d) && JL_IN_RANGE(err, l * d, d, m * d))
      for (int i = 0; i < d; ++i) v = fmaf(Pinv[j * d + i], bf16_bits_to_f32(S[l * d + i]), v);
  }
  if (JL_IN_RANGE(err, idx, 1, d * cols)) basis[idx] = __half_as_ushort(__float2half_rn(v));
}

}  // namespace dq

cudaError_t launch_dequantize_tc(const uint32_t *signs, const uint16_t *norms, int64_t n,
                                 const uint16_t *S, int m, int d, uint16_t *out,
                                 cudaStream_t stream) {
  dq::Params p{};
  p.codes = signs;
  p.norms = norms;
  p.B = S;
  p.n = n;
#define JL_CASE(MM, DD) \
  if (m == MM && d == DD) return dq::launch_t<MM, DD, 0>(p, out, stream);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_turbo_dequant_basis(const float *Pinv, const uint16_t *S, int m, int d,
                                       uint16_t *basis, cudaStream_t stream) {
  if (m != d || (d != 64 && d != 128)) return cudaErrorNotSupported;
  int *err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  const int total = d * (d + m);
  dq::turbo_basis_kernel<<<(total + dq::BASIS_THREADS - 1) / dq::BASIS_THREADS,
                           dq::BASIS_THREADS, 0, stream>>>(Pinv, S, m, d, basis, err);
  return cudaGetLastError();
}

cudaError_t launch_turbo_dequantize(const uint32_t *codes, const uint16_t *norms, int64_t n,
                                    const uint16_t *basis, int m, int d, int bits,
                                    uint16_t *out, cudaStream_t stream) {
  if (m != d || (d != 64 && d != 128)) return cudaErrorNotSupported;
  float mag[4], thr[3];
  if (!turbo_magnitudes(d, bits, mag, thr)) return cudaErrorNotSupported;
  dq::Params p{};
  p.codes = codes;
  p.norms = norms;
  p.B = basis;
  p.n = n;
  uint32_t h[4];
  for (int i = 0; i < 4; ++i) {
    h[i] = (uint32_t)__half_as_ushort(__float2half_rn(mag[i]));
    p.mag[i] = h[i] | (h[i] << 16);
  }
  p.dmag01 = h[0] ^ h[1];
  p.dmag23 = h[2] ^ h[3];
#define JL_CASE(TB, DD) \
  if (bits == TB && d == DD) return dq::launch_t<DD, DD, TB>(p, out, stream);
  JL_CASE(1, 128) JL_CASE(2, 128) JL_CASE(3, 128) JL_CASE(1, 64) JL_CASE(2, 64) JL_CASE(3, 64)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
