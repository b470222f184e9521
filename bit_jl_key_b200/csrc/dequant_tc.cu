// dequant_tc.cu -- explicit QJL dequantizer on the 5th-generation tensor cores.
//
// Dequantizer Q^-1(z) = sqrt(pi/2)/d * S^T z of "The Geometry of Forgetting:
// How Three Papers Cracked KV Cache Quantization", section "QJL: one bit, zero
// parameters, unbiased inner products", taken with m sketch rows and with the
// stored norm restoring the magnitude (same page, "PolarQuant" section):
//     khat = sqrt(pi/2)/m * ||k|| * S^T z,   z_i = +1 if code bit i is set.
// The reconstruction error E||k - khat||^2 is the page's D_mse for this
// quantizer.
//
// For a tile of 128 codes, Khat = Z S is a dense bf16 contraction (M = 128
// codes, N = d, K = m): tcgen05.mma with Z read from tensor memory, S^T from
// shared memory (128-byte swizzle, K-major) and the fp32 accumulator in
// tensor memory.
//   * Z (the A operand) is expanded from the code bits by threads straight
//     into tensor memory, one K-chunk of 64 coordinates (32 columns of bf16
//     pairs, one tcgen05.st per thread) at a time, into a ring of chunks; it
//     never passes through shared memory.  A bf16 pair holds coordinates
//     (p, p + 16) of a 32-bit code word, built with one shift and one LOP3:
//     ((w << (15 - p)) & 0x80008000) ^ 0xBF80BF80.
//   * S^T (the B operand, N = d rows of K = m) stays resident; its K order is
//     the same permutation of each 32-coordinate block, so the contraction is
//     unchanged.
//   * The epilogue scales row r by sqrt(pi/2)/m * ||k_r||, rounds to bf16,
//     writes its 32 rows into a 128-byte-swizzled staging tile in shared
//     memory and stores them with bulk-tensor copies (which also clip rows
//     past the last code).
//   * An expander thread copies its code row of the tile two ahead into a
//     shared-memory ring with cp.async while it expands the current one.
//
// One persistent CTA per SM, 13 warps with fixed roles:
//   warps 0-7  expand: warp w writes TMEM lane quadrant w % 4 (code rows
//              32 (w % 4) .. + 31 of the tile) for part w / 4 of the tile's
//              K-chunks (the first or the second half), so two warps expand
//              each row at once; each thread copies its half of its code
//              row two tiles ahead.
//   warps 8-11 epilogue: warp w reads TMEM lane quadrant w % 4.
//   warp 12    owns the TMEM allocation; one elected lane issues the MMAs of a tile
//              into one of two accumulators and commits them to the barriers
//              that free the Z chunks and publish the accumulator.
// Every mbarrier wait is bounded (about 2 s of GPU time); a wait that runs
// out records DERR_TC_WAIT_TIMEOUT, raises a shared abort flag, and the CTA
// still frees its TMEM.
#include "jl_common.cuh"
#include "jl_internal.h"

#include <cudaTypedefs.h>

namespace jlk {
namespace dq {

constexpr int BM = 128;          // codes per tile (MMA M)
constexpr int CHUNK_K = 64;      // coordinates per Z chunk
constexpr int CHUNK_COLS = CHUNK_K / 2;  // TMEM columns of a Z chunk (bf16 pairs)
constexpr int EXP_PARTS = 2;     // expander warps per TMEM lane quadrant
constexpr int EXP_WARPS = 4 * EXP_PARTS, EPI_WARPS = 4;
constexpr int MMA_WARP = EXP_WARPS + EPI_WARPS;
constexpr int THREADS = (MMA_WARP + 1) * 32;
constexpr int CODE_SLOTS = 3;    // code rows in flight: the tile and two ahead
constexpr unsigned long long WAIT_NS = WAIT_LIMIT_NS;

template <int M, int D>
struct Cfg {
  static constexpr int KCH = M / CHUNK_K;             // Z chunks per tile (>= 1)
  static constexpr int ST_CHUNK = D * 128;            // one K-chunk of S^T
  static constexpr int ST_BYTES = M * D * 2;
  // output staging: per epilogue warp, 32 rows x d bf16 as D/64 swizzled
  // boxes of 32 x 128 B; two buffers per warp when they fit beside 4 Z chunks
  static constexpr int OBOX = 32 * 128;
  static constexpr int OWARP = (D / 64) * OBOX;
  static constexpr int CODE_ROW = M / 8;              // bytes per code
  static constexpr int C_BYTES = CODE_SLOTS * BM * CODE_ROW;
  static constexpr int OBUF = 2;
  static constexpr int O_BYTES = EPI_WARPS * OBUF * OWARP;
  // tensor memory: accumulators at columns [0, 2d), Z chunks after them
  static constexpr int ACC = 2;
  static constexpr int TMEM_COLS = 512;
  static constexpr int Z_COL0 = ACC * D;
  static constexpr int RING_RAW = (TMEM_COLS - Z_COL0) / CHUNK_COLS;
  static constexpr int RING = RING_RAW > 8 ? 8 : RING_RAW;
  static constexpr int OFF_O = ST_BYTES;
  static constexpr int OFF_C = OFF_O + O_BYTES;
  static constexpr int OFF_BAR = OFF_C + C_BYTES;
  static constexpr int NBAR = 2 * RING + 2 * ACC;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + align slack
  static_assert(M % CHUNK_K == 0 && RING >= 2, "Z ring");
  static_assert(Z_COL0 + RING * CHUNK_COLS <= TMEM_COLS, "tensor memory columns");
  static constexpr int CODE_WORDS = M / 32;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct Params {
  const uint32_t *signs;  // n x m/32
  const uint16_t *norms;  // n binary16
  const uint16_t *S;      // m x d bf16
  int64_t n, num_tiles;
  float coef;             // sqrt(pi/2) / m
  int *err;
};

// --------------------------------------------------------------------------
// PTX wrappers
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// generic-proxy writes to shared memory -> visible to the tensor core
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// K-major operand, 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
// D (tensor memory) += A (tensor memory, one row per lane) * B (shared memory)
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive columns of this thread's lane <- v
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
      "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
      "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]),
      "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
        "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
        "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]),
        "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
// wait for this thread's TMEM loads, tied to the registers of one load
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]),
                 "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                 "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]),
                 "+r"(v[27]), "+r"(v[28]), "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
               :
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

// Bounded wait on a barrier phase; false when the wait ran out or another
// role gave up (then the error word is set and the shared abort flag raised).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity,
                                           volatile int *abort_flag, int *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > WAIT_NS) {
        *abort_flag = 1;
        record_device_error(err, DERR_TC_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Position of coordinate i of a 32-coordinate block in the operand's K
// order: bf16 pair j holds coordinates j (low half) and j + 16 (high half).
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

template <int M, int D>
__global__ void __launch_bounds__(THREADS, 1)
    dequant_tc_kernel(const __grid_constant__ CUtensorMap tmap_out, const Params p) {
  using C = Cfg<M, D>;
  extern __shared__ uint8_t dq_smem_raw[];
  const uint32_t raw = smem_u32(dq_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = dq_smem_raw + (base - raw);
  const uint32_t sST = base;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto zfull_bar = [&](int s) { return bar0 + 8u * s; };
  auto zempty_bar = [&](int s) { return bar0 + 8u * (C::RING + s); };
  auto afull_bar = [&](int a) { return bar0 + 8u * (2 * C::RING + a); };
  auto aempty_bar = [&](int a) { return bar0 + 8u * (2 * C::RING + C::ACC + a); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int *abort_flag =
      reinterpret_cast<volatile int *>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::RING; ++s) {
      mbar_init(zfull_bar(s), 4);          // one arrive per quadrant's expander warp
      mbar_init(zempty_bar(s), 1);         // MMA commit
    }
    for (int a = 0; a < C::ACC; ++a) {
      mbar_init(afull_bar(a), 1);          // MMA commit
      mbar_init(aempty_bar(a), EPI_WARPS); // epilogue warps
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
  // S^T into shared memory, once: 16-byte unit (row n, K positions 8u..8u+7)
  // per thread and step; K position k holds coordinate i with k_slot(i) = k
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
        h2[hh] = __ldg(p.S + (int64_t)i * D + n);
      }
      pk[q] = (uint32_t)h2[0] | ((uint32_t)h2[1] << 16);
    }
    *reinterpret_cast<uint4 *>(gbase + sw128_offset(n, 8 * u, D)) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int64_t ntiles = p.num_tiles;

  if (warp < EXP_WARPS) {
    // ---------------- expand: quadrant q = warp % 4 (row r = 32 q + lane),
    // part pt = warp / 4: chunks [kc0, kc0 + nk) of every tile; the part's
    // code words of the tile two ahead are copied meanwhile
    const int q = warp & 3, pt = warp >> 2;
    const int r = 32 * q + lane;
    constexpr int KP = (C::KCH + EXP_PARTS - 1) / EXP_PARTS;  // chunks per part
    const int kc0 = pt * KP;
    const int nk = C::KCH - kc0 < KP ? C::KCH - kc0 : KP;
    bool ok = nk > 0;
    const uint32_t pbytes = (uint32_t)(KP * 8);             // 2 code words per chunk
    const uint32_t crow = base + C::OFF_C + r * C::CODE_ROW + pt * pbytes;
    auto code_slot = [&](int slot) { return crow + (uint32_t)(slot * BM * C::CODE_ROW); };
    auto copy_part = [&](uint32_t dst, int64_t row) {
      const bool live = row < p.n && JL_IN_RANGE(p.err, row * (M / 8) + pt * pbytes, KP * 8,
                                                 p.n * (M / 8));
      const uint8_t *src = reinterpret_cast<const uint8_t *>(p.signs + (live ? row : 0) * (M / 32)) +
                           pt * pbytes;
      if constexpr (KP * 8 >= 16) {
#pragma unroll
        for (int u = 0; u < KP * 8 / 16; ++u) cp_async_16(dst + 16 * u, src + 16 * u, live ? 16 : 0);
      } else {
        cp_async_8(dst, src, live ? 8 : 0);
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
    for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      copy_part(code_slot(cs == 0 ? CODE_SLOTS - 1 : cs - 1),
                (tile + (int64_t)(CODE_SLOTS - 1) * gridDim.x) * BM + r);
      cp_async_wait<CODE_SLOTS - 1>();  // this tile's words have landed
      uint32_t cur[2 * KP];
      {
        const uint8_t *src = gbase + (code_slot(cs) - base);
#pragma unroll
        for (int i = 0; i < 2 * KP; ++i) cur[i] = reinterpret_cast<const uint32_t *>(src)[i];
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
        if (!wait_phase(zempty_bar(s), ph ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        // the chunk's 32 TMEM columns of row r: column 16 h + j holds the
        // pair (j, j + 16) of code word 2 kc + h
        uint32_t z[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t w = cur[2 * kk + half];  // rows past the end expand a zero code
#pragma unroll
          for (int j = 0; j < 16; ++j)
            z[16 * half + j] = ((w << (15 - j)) & 0x80008000u) ^ 0xBF80BF80u;
        }
        tmem_st32(tmem_base + ((uint32_t)(32 * q) << 16) +
                      (uint32_t)(C::Z_COL0 + s * CHUNK_COLS), z);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(zfull_bar(s));
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
    int64_t t = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++t) {
      const int a = (int)(t & 1);
      const uint32_t aph = (uint32_t)((t >> 1) & 1);
      const int64_t row = tile * BM + 32 * q + lane;
      const bool live = row < p.n && JL_IN_RANGE(p.err, row, 1, p.n);
      const float f = live ? p.coef * __half2float(__ushort_as_half(__ldg(p.norms + row))) : 0.f;
      const int ob = (int)(t % C::OBUF);
      uint8_t *stage = gbase + C::OFF_O + (ew * C::OBUF + ob) * C::OWARP;
      // the staging buffer's previous stores must have read it
      if (lane == 0) bulk_wait_read<C::OBUF - 1>();
      __syncwarp();
      if (!wait_phase(afull_bar(a), aph, abort_flag, p.err)) break;
      __syncwarp();
      tc_fence_after();
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
      tmem_ld32(trow, va);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 64) {
        tmem_ld_wait(va);
        tmem_ld32(trow + c0 + 32, vb);
        emit(va, c0);
        tmem_ld_wait(vb);
        if (c0 + 64 < D) tmem_ld32(trow + c0 + 64, va);
        emit(vb, c0 + 32);
      }
      tc_fence_before();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(aempty_bar(a));
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
      constexpr uint32_t idesc = (1u << 4)                  // D: fp32
                                 | (1u << 7) | (1u << 10)   // A, B: bf16
                                 | ((uint32_t)(D >> 3) << 17)   // N
                                 | ((uint32_t)(BM >> 4) << 24); // M
      const uint64_t b0 = smem_desc_sw128(sST);
      const uint32_t b_hi = (uint32_t)(b0 >> 32), b_lo0 = (uint32_t)b0;
      int rs = 0;
      uint32_t rph = 0;
      uint32_t t = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++t) {
        const int a = (int)(t & 1u);
        const uint32_t aph = (t >> 1) & 1u;
        if (!__all_sync(0xffffffffu, wait_phase(aempty_bar(a), aph ^ 1u, abort_flag, p.err)))
          break;
        tc_fence_after();
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
          tc_fence_after();
          uint32_t el;
          asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.u32 %0, 1, 0, e;\n}\n"
                       : "=r"(el));
          if (el) {
            const uint32_t blo = b_lo0 + (uint32_t)kc * (uint32_t)(C::ST_CHUNK >> 4);
#pragma unroll
            for (int kk = 0; kk < CHUNK_K / 16; ++kk) {  // K = 16: 8 columns of A
              const uint32_t atm = tmem_base + (uint32_t)(C::Z_COL0 + s * CHUNK_COLS + kk * 8);
              const uint64_t bdesc = ((uint64_t)b_hi << 32) | (uint64_t)(blo + (uint32_t)(kk * 2));
              mma_bf16_ts(tmem_base + a * D, atm, bdesc, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(zempty_bar(s));
          }
          __syncwarp();
        }
        if (!ok) break;
        uint32_t el2;
        asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.u32 %0, 1, 0, e;\n}\n"
                     : "=r"(el2));
        if (el2) mma_commit(afull_bar(a));
        __syncwarp();
      }
      // drain: the last accumulator's MMAs must be complete before TMEM is freed
      if (t > 0 && ok && lane == 0) {
        const uint32_t tl = t - 1;
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(afull_bar((int)(tl & 1u)), (tl >> 1) & 1u) &&
               globaltimer() - t0 < WAIT_NS) {
        }
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
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

template <int M, int D>
cudaError_t launch_t(const uint32_t *signs, const uint16_t *norms, int64_t n,
                     const uint16_t *S, uint16_t *out, cudaStream_t stream) {
  using C = Cfg<M, D>;
  int *err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  CUtensorMap tmap;
  if (!make_out_map(&tmap, out, n, D)) return cudaErrorInvalidValue;
  Params p{signs, norms, S, n, (n + BM - 1) / BM,
           (float)(1.2533141373155002512 / (double)M), err};
  cudaError_t e = cudaFuncSetAttribute(dequant_tc_kernel<M, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t sms = device_sm_count();
  const int64_t grid = p.num_tiles < sms ? p.num_tiles : sms;
  dequant_tc_kernel<M, D><<<(int)grid, THREADS, C::SMEM, stream>>>(tmap, p);
  return cudaGetLastError();
}

}  // namespace dq

cudaError_t launch_dequantize_tc(const uint32_t *signs, const uint16_t *norms, int64_t n,
                                 const uint16_t *S, int m, int d, uint16_t *out,
                                 cudaStream_t stream) {
#define JL_CASE(MM, DD) \
  if (m == MM && d == DD) return dq::launch_t<MM, DD>(signs, norms, n, S, out, stream);
  JL_CASE(64, 64) JL_CASE(128, 64) JL_CASE(256, 64) JL_CASE(512, 64)
  JL_CASE(64, 128) JL_CASE(128, 128) JL_CASE(256, 128) JL_CASE(512, 128)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
