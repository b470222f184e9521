// turbo_tc.cu -- TurboQuant-prod keys: codebook, rotation, quantizer.
//
// "The Geometry of Forgetting: How Three Papers Cracked KV Cache
// Quantization":
//  * section "Random rotation, and what high dimensions do to your
//    intuitions": Pi from orthogonalising a Gaussian matrix; a coordinate of a
//    rotated unit vector has the density
//        f(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2);
//  * section "TurboQuant: bridging MSE and inner product, in two stages": the
//    Lloyd-Max codebook of f for the first b-1 bits of every rotated
//    coordinate, then QJL on the residual.
//
// Codebook (host, float64, once per (d, bits)): Lloyd's two conditions
// alternated on the positive half of the even density -- boundaries at the
// midpoints of neighbouring centroids, each centroid the mean of f over its
// cell.  Cell masses by composite Gauss-Legendre quadrature of f, first
// moments from the antiderivative of x (1 - x^2)^((d-3)/2).
//
// Rotation (device, float64, init time): G from the sketch generator,
// Gram-Schmidt column by column with one re-orthogonalisation pass (the
// positive-diagonal QR factor), rounded to bf16; then the inverse of the bf16
// matrix by Newton-Schulz iterations X <- X (2I - Pi X) from X = Pi^T.
//
// Quantizer (tensor cores), per tile of 128 keys:
//   MMA 1   D = K Pi^T             (K: TMA-loaded bf16 tile; Pi resident)
//   epilogue A  (one thread per key): y = D / ||k||; cells by
//           a branch-free search of |y| over the positive boundaries (the cell
//           bits are the code's planes); r = y - c[cell], ||r||, and
//           rt = bf16(r) written to tensor memory as the A operand of
//   MMA 2   D = rt S^T             (S resident; D reuses MMA 1's columns)
//   epilogue B  sign words of D.
// Warp roles: 0 TMA producer, 1 MMA issuer, 2-9 epilogue: warp w reads TMEM
// lane quadrant w % 4 (32 keys, whole rows) of the tiles of parity
// (w - 2) / 4, running A then B of each.  The two epilogue warps that share a
// quadrant (and a scheduler) thus work on different tiles and need no
// exchange; one hides the other's waits.  Tensor memory: MMA 1 results and
// residual rows double-buffered by tile parity, MMA 2 results single-buffered
// (MMA 2 of a tile waits for epilogue B of the previous one, which the other
// warp runs right after its A).  Every wait is bounded; a
// wait that runs out records DERR_TC_WAIT_TIMEOUT, tells the other roles to
// stop, and the CTA drains its copies and frees its tensor memory.
#include "jl_common.cuh"
#include "jl_internal.h"
#include "jl_rng.cuh"
#include "jl_tc.cuh"

#include <cudaTypedefs.h>
#include <math.h>

#include <map>
#include <mutex>
#include <utility>
#include <vector>

namespace jlk {
namespace turbo {

// --------------------------------------------------------------------------
// codebook (host)

struct GaussLegendre {
  std::vector<double> x, w;  // nodes and weights on [-1, 1]
  explicit GaussLegendre(int n) : x(n), w(n) {
    // Newton's method on the Legendre polynomial P_n from the Chebyshev-like
    // initial guesses cos(pi (i + 3/4) / (n + 1/2))
    for (int i = 0; i < (n + 1) / 2; ++i) {
      double z = cos(M_PI * (i + 0.75) / (n + 0.5)), dp = 0.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        dp = n * (z * p1 - p0) / (z * z - 1.0);
        const double dz = p1 / dp;
        z -= dz;
        if (fabs(dz) < 1e-16) break;
      }
      x[i] = -z;
      x[n - 1 - i] = z;
      w[i] = w[n - 1 - i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

struct Density {
  int d;
  double logc;  // log of Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))
  explicit Density(int dd)
      : d(dd), logc(lgamma(dd / 2.0) - 0.5 * log(M_PI) - lgamma((dd - 1) / 2.0)) {}
  double f(double x) const {
    const double s = 1.0 - x * x;
    if (s <= 0.0) return d == 3 ? exp(logc) : 0.0;
    return exp(logc + 0.5 * (d - 3) * log(s));
  }
  // int_lo^hi x f(x) dx
  double moment(double lo, double hi) const {
    auto F = [&](double x) {
      const double s = 1.0 - x * x;
      return s <= 0.0 ? 0.0 : -exp(0.5 * (d - 1) * log(s)) / (d - 1);
    };
    return exp(logc) * (F(hi) - F(lo));
  }
  // int_lo^hi f(x) dx: composite Gauss-Legendre over panels of width <=
  // 1/(8 sqrt(d)) (a fraction of the density's spread)
  double mass(double lo, double hi, const GaussLegendre &gl) const {
    // beyond 15 standard deviations (1/sqrt(d) each) f is below e^-110 of its
    // peak: leave that tail out of the panels
    hi = fmin(hi, fmax(0.0, 15.0 / sqrt((double)d)));
    const double width = hi - lo;
    if (width <= 0.0) return 0.0;
    const double pw = 0.125 / sqrt((double)d);
    const int panels = (int)ceil(width / pw) < 1 ? 1 : (int)ceil(width / pw);
    const double h = width / panels;
    double s = 0.0;
    for (int p = 0; p < panels; ++p) {
      const double a = lo + p * h, mid = a + 0.5 * h;
      double ps = 0.0;
      for (size_t k = 0; k < gl.x.size(); ++k) ps += gl.w[k] * f(mid + 0.5 * h * gl.x[k]);
      s += 0.5 * h * ps;
    }
    return s;
  }
};

// Positive half a_0 < ... < a_{H-1} of the symmetric L = 2H-level quantizer.
static std::vector<double> lloyd_max_half(int d, int bits) {
  const int H = 1 << (bits - 1);
  const Density den(d);
  const GaussLegendre gl(16);
  std::vector<double> a(H), t(H + 1);
  const double sd = 1.0 / sqrt((double)d);
  for (int i = 0; i < H; ++i) a[i] = fmin((i + 0.5) * 2.5 * sd / H, 1.0 - (H - i) * 1e-3);
  // stop once a sweep moves no centroid by more than 1e-14 of the largest
  // (far below the float rounding of the result)
  for (int it = 0; it < 100000; ++it) {
    t[0] = 0.0;
    t[H] = 1.0;
    for (int i = 1; i < H; ++i) t[i] = 0.5 * (a[i - 1] + a[i]);
    double move = 0.0;
    for (int i = 0; i < H; ++i) {
      const double nm = den.moment(t[i], t[i + 1]) / den.mass(t[i], t[i + 1], gl);
      move = fmax(move, fabs(nm - a[i]));
      a[i] = nm;
    }
    if (move <= 1e-14 * a[H - 1]) break;
  }
  return a;
}

struct Codebook {
  int L = 0;
  double c[8];      // centroids, ascending
  float cf[8];      // as float
  float thr[7];     // float((c_i + c_{i+1}) / 2)
  double walsh[4];  // odd Walsh terms: single planes, then (3 bits) all three
};

static const Codebook *codebook(int d, int bits) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, Codebook> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(d, bits);
  auto it = cache.find(key);
  if (it != cache.end()) return &it->second;
  const std::vector<double> a = lloyd_max_half(d, bits);
  Codebook cb;
  const int H = (int)a.size();
  cb.L = 2 * H;
  for (int i = 0; i < H; ++i) {
    cb.c[H + i] = a[i];
    cb.c[H - 1 - i] = -a[i];
  }
  for (int j = 0; j < cb.L; ++j) cb.cf[j] = (float)cb.c[j];
  for (int j = 0; j + 1 < cb.L; ++j) cb.thr[j] = (float)(0.5 * (cb.c[j] + cb.c[j + 1]));
  // Walsh coefficients (1/L) sum_j c_j prod_{p in S} e_p(j), e_p = +-1 from
  // bit p of j, for the odd subsets S (the even ones vanish for a symmetric
  // codebook): {p} for each plane, then {0, 1, 2} with three planes
  auto walsh_of = [&](int mask) {
    double s = 0.0;
    for (int j = 0; j < cb.L; ++j) {
      double e = 1.0;
      for (int p = 0; p < bits; ++p)
        if ((mask >> p) & 1) e *= ((j >> p) & 1) ? 1.0 : -1.0;
      s += cb.c[j] * e;
    }
    return s / cb.L;
  };
  for (int k = 0; k < 4; ++k) cb.walsh[k] = 0.0;
  for (int p = 0; p < bits; ++p) cb.walsh[p] = walsh_of(1 << p);
  if (bits == 3) cb.walsh[3] = walsh_of(7);
  return &cache.emplace(key, cb).first->second;
}

// --------------------------------------------------------------------------
// rotation (device, float64)

constexpr int ROT_THREADS = 256;

// One CTA.  Shared memory: Qc (column j of Q contiguous), v, r.
template <int D>
__global__ void __launch_bounds__(ROT_THREADS) rot_gram_schmidt_kernel(uint64_t seed,
                                                                        uint16_t *Pi,
                                                                        double *Pit64) {
  extern __shared__ double rot_smem[];
  double *Qc = rot_smem;        // [D][D]
  double *v = Qc + D * D;       // [D]
  double *r = v + D;            // [D]
  double *red = r + D;          // [ROT_THREADS / 32]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = ROT_THREADS / 32;
  for (int j = 0; j < D; ++j) {
    if (tid < D) v[tid] = gauss_at(seed, (uint64_t)tid * D + j);  // G[tid][j]
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      // r_i = <q_i, v> for i < j
      for (int i = warp; i < j; i += NW) {
        double s = 0.0;
        for (int k = lane; k < D; k += 32) s += Qc[i * D + k] * v[k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) r[i] = s;
      }
      __syncthreads();
      if (tid < D) {
        double s = 0.0;
        for (int i = 0; i < j; ++i) s += Qc[i * D + tid] * r[i];
        v[tid] -= s;
      }
      __syncthreads();
    }
    double s = tid < D ? v[tid] * v[tid] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[warp] = s;
    __syncthreads();
    double nn = 0.0;
    for (int w = 0; w < NW; ++w) nn += red[w];
    const double inv = 1.0 / sqrt(nn);
    if (tid < D) Qc[j * D + tid] = v[tid] * inv;
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += ROT_THREADS) {
    const int i = e / D, j = e - i * D;  // Pi[i][j] = Q[i][j] = Qc[j][i]
    const uint16_t b = bf16_from_f64_bits(Qc[j * D + i]);
    Pi[e] = b;
    Pit64[e] = (double)__uint_as_float((uint32_t)b << 16);
  }
}

// out = alpha * A B + beta * C  (n x n, row-major float64); 16 x 16 tiles
__global__ void rot_gemm_kernel(const double *A, const double *B, const double *C,
                                double alpha, double beta, double *out, int n) {
  __shared__ double ta[16][17], tb[16][17];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int row = blockIdx.y * 16 + ty, col = blockIdx.x * 16 + tx;
  double s = 0.0;
  for (int k0 = 0; k0 < n; k0 += 16) {
    ta[ty][tx] = A[row * n + k0 + tx];
    tb[ty][tx] = B[(k0 + ty) * n + col];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) s += ta[ty][k] * tb[k][tx];
    __syncthreads();
  }
  out[row * n + col] = alpha * s + (C ? beta * C[row * n + col] : 0.0);
}

__global__ void rot_transpose_kernel(const double *A, double *out, int n) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n * n) {
    const int i = e / n, j = e - i * n;
    out[j * n + i] = A[e];
  }
}

__global__ void rot_to_f32_kernel(const double *A, float *out, int n) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n * n) out[e] = (float)A[e];
}

constexpr int NS_ITERS = 6;

size_t rotation_workspace_bytes(int d) {
  if (d != 64 && d != 128) return 0;
  return 4 * (size_t)d * d * sizeof(double);
}

cudaError_t launch_rotation(uint16_t *Pi, float *Pinv, int d, uint64_t seed, void *ws,
                            cudaStream_t stream) {
  double *P64 = reinterpret_cast<double *>(ws);
  double *X = P64 + (size_t)d * d, *Xn = X + (size_t)d * d, *T = Xn + (size_t)d * d;
  const size_t smem = ((size_t)d * d + 2 * d + ROT_THREADS / 32) * sizeof(double);
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(rot_gram_schmidt_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rot_gram_schmidt_kernel<128><<<1, ROT_THREADS, smem, stream>>>(seed, Pi, P64);
  } else {
    rot_gram_schmidt_kernel<64><<<1, ROT_THREADS, smem, stream>>>(seed, Pi, P64);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nn = d * d;
  rot_transpose_kernel<<<(nn + 255) / 256, 256, 0, stream>>>(P64, X, d);
  const dim3 g(d / 16, d / 16), b(16, 16);
  for (int it = 0; it < NS_ITERS; ++it) {
    rot_gemm_kernel<<<g, b, 0, stream>>>(P64, X, nullptr, 1.0, 0.0, T, d);  // T = Pi X
    rot_gemm_kernel<<<g, b, 0, stream>>>(X, T, X, -1.0, 2.0, Xn, d);        // 2X - X T
    double *tmp = X;
    X = Xn;
    Xn = tmp;
  }
  rot_to_f32_kernel<<<(nn + 255) / 256, 256, 0, stream>>>(X, Pinv, d);
  return cudaGetLastError();
}

// --------------------------------------------------------------------------
// quantizer (tensor cores), d = m = 64 or 128

constexpr int BM = 128;

// TB cell planes, head dim D = rotation size = residual sketch rows M
template <int TB, int D>
struct QCfg {
  static constexpr int M = D;
  static constexpr int KCH = D / 64;
  static constexpr int A_CHUNK = BM * 128;      // one 64-column swizzle column of a tile
  static constexpr int A_STAGE = BM * D * 2;    // 32 or 16 KB
  static constexpr int PI_CHUNK = D * 128;      // D rows x 64 columns of Pi
  static constexpr int S_CHUNK = M * 128;       // M rows x 64 columns of S
  static constexpr int PI_BYTES = D * D * 2;
  static constexpr int S_BYTES = M * D * 2;
  static constexpr int STAGES = 4;
  static constexpr int EPI_WARPS = 8;           // two per TMEM lane quadrant (tile parities)
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  static constexpr int OFF_PI = 0;
  static constexpr int OFF_S = PI_BYTES;
  static constexpr int OFF_A = PI_BYTES + S_BYTES;
  static constexpr int OFF_BAR = OFF_A + STAGES * A_STAGE;
  static constexpr int NBAR = 2 * STAGES + 2 + 2 + 2 + 1 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr int WORDS = TB * D / 32 + M / 32;
  static constexpr int PW = D / 32;             // words per plane
  static constexpr int TMEM_COLS = 4 * D;       // 512 or 256
  static constexpr int D1_COL = 0;              // rotated keys, two buffers of D columns
  static constexpr int D2_COL = 2 * D;          // residual projections, one buffer of M
  static constexpr int A2_COL = 2 * D + M;      // bf16 residual rows, two buffers of D / 2
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(OFF_S % 1024 == 0 && OFF_A % 1024 == 0, "swizzle atoms");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(STAGES % 2 == 0, "a stage holds tiles of one parity");
};

struct QParams {
  int64_t n;
  int64_t num_tiles;
  uint32_t *codes;
  uint32_t *norms;  // (||k|| | ||r|| << 16) binary16 pairs
  int *err;
  float mag[4];      // centroid magnitudes a_0 < ... (positive half of the codebook)
  float pos_thr[3];  // positive boundaries between them
};

// Odd-symmetric cells.  With H = 2^(TB-1) centroid magnitudes a_0 < ... <
// a_{H-1} (the positive half of the codebook) and the positive boundaries
// p_0 < ... < p_{H-2} between them, a coordinate y lies in magnitude cell
// mu = #{p_j < |y|} (a value on a boundary stays inward) on the side of its
// sign (0 counts as negative), i.e. cell H + mu for y > 0 and H - 1 - mu
// otherwise; its centroid is +-a_mu.  In bits: the top plane is [y > 0] and
// plane k < TB-1 is bit k of mu when y > 0 and its complement otherwise, i.e.
// XNOR(bit k of mu, [y > 0]).
//
// Every bit is the sign bit of a float, gathered into code words by funnel
// shifts: [y > 0] = sign(-y) with -y formed as D (-1/||k||) + 0, which turns
// -0 into +0, and bit k of mu = sign(p - |y|) for the boundary p of that
// search level.  The plane word is then the complement of the XOR of the two
// sign words (one logic op per 32 coordinates).
struct Magnitudes {
  float a[4];  // centroid magnitudes
  float p[3];  // positive boundaries
};

template <int TB>
struct PlaneChains {
  uint32_t top[4];          // [y > 0], four chains of 8 bits
  uint32_t mag[TB - 1 > 0 ? TB - 1 : 1][4];  // [p < |y|] of each search level
};

// -y = d * ninv + 0 with one rounding (ninv = -1/||k||): the product rounded
// as y = d / ||k|| is, negated, and a -0 product becomes +0
__device__ __forceinline__ float neg_scaled(float d, float ninv) {
  float r;
  asm("fma.rn.f32 %0, %1, %2, 0f00000000;\n" : "=f"(r) : "f"(d), "f"(ninv));
  return r;
}

// Two fp32 lanes in one 64-bit register (Blackwell's packed fp32 pipe:
// one instruction rounds each lane exactly as the scalar form would).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// magnitude of the centroid of -y = neg (pushing the magnitude bits of its
// search levels into chain g)
template <int TB>
__device__ __forceinline__ float cell_magnitude(float neg, const Magnitudes &mg,
                                                PlaneChains<TB> &ch, int g) {
  const float ay = fabsf(neg);
  if constexpr (TB == 1) {
    return mg.a[0];
  } else if constexpr (TB == 2) {
    const float d0 = mg.p[0] - ay;
    ch.mag[0][g] = __funnelshift_l(__float_as_uint(d0), ch.mag[0][g], 1);
    return d0 < 0.f ? mg.a[1] : mg.a[0];
  } else {
    const float d1 = mg.p[1] - ay;
    const bool m1 = d1 < 0.f;
    const float d0 = (m1 ? mg.p[2] : mg.p[0]) - ay;
    ch.mag[1][g] = __funnelshift_l(__float_as_uint(d1), ch.mag[1][g], 1);
    ch.mag[0][g] = __funnelshift_l(__float_as_uint(d0), ch.mag[0][g], 1);
    const bool m0 = d0 < 0.f;
    return m1 ? (m0 ? mg.a[3] : mg.a[2]) : (m0 ? mg.a[1] : mg.a[0]);
  }
}

// Cell and residual of the adjacent coordinates (jj, jj + 1) of chain g with
// packed fp32 arithmetic: -y of both from one fma, both residuals from one
// subtraction (the centroid carries the sign of y, so y - c = +-a - neg),
// and both squares into the residual norm's two lanes; the bits go into the
// chains higher coordinate first, as the scalar order does.  Returns the
// residual pair (lane 0: coordinate jj).
template <int TB>
__device__ __forceinline__ uint64_t cell_residual_pair(uint64_t d2, uint64_t ninv2,
                                                       const Magnitudes &mg, PlaneChains<TB> &ch,
                                                       int g, uint64_t &rs2) {
  const uint64_t neg2 = f32x2_fma(d2, ninv2, 0ull);  // + (+0, +0): a -0 product becomes +0
  float n0, n1;
  f32x2_unpack(neg2, n0, n1);
  ch.top[g] = __funnelshift_l(__float_as_uint(n1), ch.top[g], 1);
  const float a1 = cell_magnitude<TB>(n1, mg, ch, g);
  ch.top[g] = __funnelshift_l(__float_as_uint(n0), ch.top[g], 1);
  const float a0 = cell_magnitude<TB>(n0, mg, ch, g);
  const float s0 = __uint_as_float(__float_as_uint(a0) | (__float_as_uint(n0) & 0x80000000u));
  const float s1 = __uint_as_float(__float_as_uint(a1) | (__float_as_uint(n1) & 0x80000000u));
  const uint64_t rr2 = f32x2_sub(f32x2_pack(s0, s1), neg2);
  rs2 = f32x2_fma(rr2, rr2, rs2);
  return rr2;
}

template <int TB, int D>
__global__ void __launch_bounds__(QCfg<TB, D>::THREADS, 1)
    turbo_quantize_kernel(const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_pi,
                          const __grid_constant__ CUtensorMap tmap_s, const QParams p) {
  using C = QCfg<TB, D>;
  extern __shared__ uint8_t tq_smem_raw[];
  const uint32_t raw = smem_u32(tq_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = tq_smem_raw + (base - raw);
  const uint32_t sPi = base + C::OFF_PI, sS = base + C::OFF_S, sA = base + C::OFF_A;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto kfull = [&](int s) { return bar0 + 8u * s; };
  auto kempty = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto d1full = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
  auto afull = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 2 + a); };
  // MMA 2 of tile u commits to d2full(u & 1), waited on only by the warps of
  // that parity (so each of them sees every phase of it)
  auto d2full = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 4 + a); };
  const uint32_t d2empty = bar0 + 8u * (2 * C::STAGES + 6);
  const uint32_t wfull = bar0 + 8u * (2 * C::STAGES + 7);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int *abort_flag =
      reinterpret_cast<volatile int *>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(kfull(s), 1);
      mbar_init(kempty(s), 1 + C::EPI_WARPS / 2);  // MMA commit + the parity's warps (norms)
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(d1full(a), 1);
      mbar_init(afull(a), C::EPI_WARPS / 2);
      mbar_init(d2full(a), 1);
    }
    mbar_init(d2empty, C::EPI_WARPS / 2);
    mbar_init(wfull, 1);
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
  tcx::fence_before();
  __syncthreads();
  tcx::fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // tiles of this CTA: blockIdx.x + t * gridDim.x, t < cnt
  const int64_t cnt =
      p.num_tiles > blockIdx.x ? (p.num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      mbar_expect_tx(wfull, C::PI_BYTES + C::S_BYTES);
      for (int kc = 0; kc < C::KCH; ++kc) {
        tma_load_2d(sPi + kc * C::PI_CHUNK, &tmap_pi, kc * 64, 0, wfull);
        tma_load_2d(sS + kc * C::S_CHUNK, &tmap_s, kc * 64, 0, wfull);
      }
      int64_t t = 0;
      for (; t < cnt; ++t) {
        const int s = (int)(t % C::STAGES);
        const uint32_t ph = (uint32_t)((t / C::STAGES) & 1);
        if (!tcx::wait_phase(kempty(s), ph ^ 1u, abort_flag, p.err)) break;
        const int64_t tile = blockIdx.x + t * gridDim.x;
        mbar_expect_tx(kfull(s), C::A_STAGE);
        for (int kc = 0; kc < C::KCH; ++kc)
          tma_load_2d(sA + s * C::A_STAGE + kc * C::A_CHUNK, &tmap_k, kc * 64,
                      (int)(tile * BM), kfull(s));
      }
      for (int64_t j = (t > C::STAGES ? t - C::STAGES : 0); j < t; ++j)
        tcx::drain_wait(kfull((int)(j % C::STAGES)), (uint32_t)((j / C::STAGES) & 1));
      tcx::drain_wait(wfull, 0);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: MMA 1 of tile t, then MMA 2 of tile t - 1.
    // The whole warp runs the loop (waits and counters warp-uniform) and one
    // elected lane issues; descriptors are the base plus a 32-bit start-address
    // add (every operand lies below 256 KB of shared memory).
    {
      constexpr uint32_t idesc = tcx::idesc_f16(BM, D, 1);  // N = D = M
      const uint64_t da = tcx::desc_sw128(sA), dpi = tcx::desc_sw128(sPi), ds = tcx::desc_sw128(sS);
      const uint32_t a_hi = (uint32_t)(da >> 32), a_lo0 = (uint32_t)da;
      const uint32_t pi_hi = (uint32_t)(dpi >> 32), pi_lo = (uint32_t)dpi;
      const uint32_t s_hi = (uint32_t)(ds >> 32), s_lo = (uint32_t)ds;
      bool ok = __all_sync(0xffffffffu, tcx::wait_phase(wfull, 0, abort_flag, p.err));
      int64_t issued2 = 0;
      int ks = 0;          // key stage of tile t and the phase it completes next
      uint32_t kph = 0;
      for (int64_t t = 0; ok && t <= cnt; ++t) {
        if (t < cnt) {
          const int s = ks;
          const int a = (int)(t & 1);
          // the key tile has landed; accumulator a was read by epilogue A of t - 2
          const bool got = tcx::wait_phase(kfull(s), kph, abort_flag, p.err) &&
                           (t < 2 || tcx::wait_phase(afull(a), (uint32_t)(((t - 2) >> 1) & 1),
                                                     abort_flag, p.err));
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          tcx::fence_after();
          if (tcx::elect_one()) {
            const uint32_t alo = a_lo0 + (uint32_t)s * (uint32_t)(C::A_STAGE >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off =
                  ((uint32_t)(kk >> 2) * (uint32_t)C::A_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
              const uint32_t woff =
                  ((uint32_t)(kk >> 2) * (uint32_t)C::PI_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
              const uint64_t ad = ((uint64_t)a_hi << 32) | (uint64_t)(alo + off);
              const uint64_t bd = ((uint64_t)pi_hi << 32) | (uint64_t)(pi_lo + woff);
              tcx::mma_ss(tmem_base + C::D1_COL + a * D, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            tcx::commit(d1full(a));
            tcx::commit(kempty(s));
          }
          __syncwarp();
          if (++ks == C::STAGES) {
            ks = 0;
            kph ^= 1u;
          }
        }
        if (t >= 1) {
          const int64_t u = t - 1;
          const int a = (int)(u & 1);
          // residual rows of u written; the projection buffer read by B of u - 1
          const bool got = tcx::wait_phase(afull(a), (uint32_t)((u >> 1) & 1), abort_flag, p.err) &&
                           tcx::wait_phase(d2empty, (uint32_t)((u & 1) ^ 1), abort_flag, p.err);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          tcx::fence_after();
          if (tcx::elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t woff =
                  ((uint32_t)(kk >> 2) * (uint32_t)C::S_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
              const uint64_t bd = ((uint64_t)s_hi << 32) | (uint64_t)(s_lo + woff);
              tcx::mma_ts(tmem_base + C::D2_COL, tmem_base + C::A2_COL + a * (D / 2) + kk * 8, bd,
                          idesc, kk > 0 ? 1u : 0u);
            }
            tcx::commit(d2full(a));
          }
          __syncwarp();
          ++issued2;
        }
      }
      // the last products must be complete before tensor memory is freed
      if (issued2 > 0 && lane == 0)
        tcx::drain_wait(d2full((int)((issued2 - 1) & 1)), (uint32_t)(((issued2 - 1) >> 1) & 1));
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: key row r = 32 (warp % 4) + lane of the
    // tiles of parity h
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const int r = 32 * q + lane;
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16);
    Magnitudes mg;
#pragma unroll
    for (int i = 0; i < 4; ++i) mg.a[i] = p.mag[i];
#pragma unroll
    for (int i = 0; i < 3; ++i) mg.p[i] = p.pos_thr[i];
    for (int64_t it = h; it < cnt; it += 2) {
      // ---- A: norm, cells, residual (tile it uses stage s, buffers h)
      const int s = (int)(it % C::STAGES);
      const int64_t row = (blockIdx.x + it * gridDim.x) * BM + r;
      if (!tcx::wait_phase(kfull(s), (uint32_t)((it / C::STAGES) & 1), abort_flag, p.err))
        break;
      float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
      for (int kc = 0; kc < C::KCH; ++kc) {
        const uint8_t *rowp = gbase + C::OFF_A + s * C::A_STAGE + kc * C::A_CHUNK + r * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4 *>(rowp + ((ch ^ (r & 7)) << 4));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) bf16x2_sq_acc(w4[e], ss0, ss1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(kempty(s));
      const float nk = sqrtf(ss0 + ss1);
      const float ninv = nk > 0.f ? -1.f / nk : -0.f;
      if (!tcx::wait_phase(d1full(h), (uint32_t)((it >> 1) & 1), abort_flag, p.err)) break;
      __syncwarp();
      tcx::fence_after();
      uint32_t planes[TB][2];
      uint64_t rs2 = 0ull;                       // residual sum of squares, two lanes
      const uint64_t ninv2 = f32x2_pack(ninv, ninv);
      uint32_t va[32], vb[32];
      const uint32_t dcol = tq + (uint32_t)(C::D1_COL + h * D);
      const uint32_t acol = tq + (uint32_t)(C::A2_COL + h * (D / 2));
      auto chunk = [&](uint32_t (&v)[32], int ch) {
        PlaneChains<TB> pc;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          pc.top[g] = 0u;
#pragma unroll
          for (int k = 0; k < (TB > 1 ? TB - 1 : 1); ++k) pc.mag[k][g] = 0u;
        }
        // coordinates 8 g + jj and 8 g + jj + 1, highest first so that the
        // funnel shifts leave bit jj of chain g at position jj
#pragma unroll
        for (int jj = 6; jj >= 0; jj -= 2)
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int e = 8 * g + jj;
            const uint64_t rr2 = cell_residual_pair<TB>(
                f32x2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), ninv2, mg, pc, g,
                rs2);
            float r0, r1;
            f32x2_unpack(rr2, r0, r1);
            v[e] = __float_as_uint(r0);
            v[e + 1] = __float_as_uint(r1);
          }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pk[e >> 1] = pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        tcx::st16(acol + 16 * ch, pk);
        const uint32_t top =
            pc.top[0] | (pc.top[1] << 8) | (pc.top[2] << 16) | (pc.top[3] << 24);
        planes[TB - 1][ch & 1] = top;
#pragma unroll
        for (int k = 0; k < TB - 1; ++k)
          planes[k][ch & 1] = ~(top ^ (pc.mag[k][0] | (pc.mag[k][1] << 8) |
                                       (pc.mag[k][2] << 16) | (pc.mag[k][3] << 24)));
      };
      // D / 32 chunks of 32 columns, two per pass (a rolled loop keeps the
      // code small); the second chunk's load is in flight during the first
      uint32_t *dst = p.codes + row * C::WORDS;
#pragma unroll 1
      for (int half = 0; half < D / 64; ++half) {
        tcx::ld32(dcol + 64 * half, va);
        tcx::ld32(dcol + 64 * half + 32, vb);
        tcx::ld_wait(va);
        chunk(va, 2 * half);
        tcx::ld_wait(vb);
        chunk(vb, 2 * half + 1);
        if (row < p.n &&
            JL_IN_RANGE(p.err, row * C::WORDS + 2 * half, (TB - 1) * C::PW + 2, p.n * C::WORDS)) {
#pragma unroll
          for (int pp = 0; pp < TB; ++pp)
            *reinterpret_cast<uint2 *>(dst + pp * C::PW + 2 * half) =
                make_uint2(planes[pp][0], planes[pp][1]);
        }
      }
      tcx::st_wait();
      tcx::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(afull(h));
      if (row < p.n && JL_IN_RANGE(p.err, row, 1, p.n)) {
        const uint32_t n16 = __half_as_ushort(__float2half_rn(nk));
        float rs0, rs1;
        f32x2_unpack(rs2, rs0, rs1);
        const uint32_t r16 = __half_as_ushort(__float2half_rn(sqrtf(rs0 + rs1)));
        p.norms[row] = n16 | (r16 << 16);
      }
      // ---- B: residual sign words of tile it
      if (!tcx::wait_phase(d2full(h), (uint32_t)((it >> 1) & 1), abort_flag, p.err)) break;
      __syncwarp();
      tcx::fence_after();
#pragma unroll 1
      for (int half = 0; half < C::M / 64; ++half) {
        const uint32_t d2 = tq + (uint32_t)(C::D2_COL + 64 * half);
        tcx::ld32(d2, va);
        tcx::ld32(d2 + 32, vb);
        tcx::ld_wait(va);
        const uint32_t w0 = tcx::sign_word(va);
        tcx::ld_wait(vb);
        const uint32_t w1 = tcx::sign_word(vb);
        if (row < p.n &&
            JL_IN_RANGE(p.err, row * C::WORDS + TB * C::PW + 2 * half, 2, p.n * C::WORDS))
          *reinterpret_cast<uint2 *>(dst + TB * C::PW + 2 * half) = make_uint2(w0, w1);
      }
      tcx::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(d2empty);
    }
  }

  tcx::fence_before();
  __syncthreads();
  if (warp == 1) {
    tcx::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem_base),
                 "n"(C::TMEM_COLS)
                 : "memory");
  }
}

template <int TB, int D>
static cudaError_t launch_quantize_t(const uint16_t *K, int64_t n, int64_t ldk,
                                     const uint16_t *Pi, const uint16_t *S, const Codebook &cb,
                                     uint32_t *codes, uint16_t *norms, cudaStream_t stream) {
  using C = QCfg<TB, D>;
  CUtensorMap mk, mpi, ms;
  if (!tc::make_map(&mk, K, (uint64_t)n, D, (uint64_t)ldk, BM) ||
      !tc::make_map(&mpi, Pi, D, D, D, D) || !tc::make_map(&ms, S, C::M, D, D, C::M))
    return cudaErrorInvalidValue;
  QParams p{};
  p.n = n;
  p.num_tiles = (n + BM - 1) / BM;
  p.codes = codes;
  p.norms = reinterpret_cast<uint32_t *>(norms);
  p.err = device_error_ptr();
  if (!p.err) return cudaErrorInvalidSymbol;
  const int H = cb.L / 2;
  for (int i = 0; i < 4; ++i) p.mag[i] = i < H ? cb.cf[H + i] : 0.f;
  for (int i = 0; i < 3; ++i) p.pos_thr[i] = i + 1 < H ? cb.thr[H + i] : 0.f;
  cudaError_t e = cudaFuncSetAttribute(turbo_quantize_kernel<TB, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.num_tiles < device_sm_count() ? p.num_tiles : device_sm_count();
  turbo_quantize_kernel<TB, D><<<(int)grid, C::THREADS, C::SMEM, stream>>>(mk, mpi, ms, p);
  return cudaGetLastError();
}

}  // namespace turbo

bool turbo_codebook(int d, int bits, float *centroids, double *walsh) {
  if (d < 3 || d > 4096 || bits < 1 || bits > 3) return false;
  const turbo::Codebook *cb = turbo::codebook(d, bits);
  if (centroids)
    for (int j = 0; j < cb->L; ++j) centroids[j] = cb->cf[j];
  if (walsh)
    for (int p = 0; p < 4; ++p) walsh[p] = cb->walsh[p];
  return true;
}

bool turbo_magnitudes(int d, int bits, float *mag, float *pos_thr) {
  if (d < 3 || d > 4096 || bits < 1 || bits > 3) return false;
  const turbo::Codebook *cb = turbo::codebook(d, bits);
  const int H = cb->L / 2;
  for (int i = 0; i < 4; ++i) mag[i] = i < H ? cb->cf[H + i] : 0.f;
  for (int i = 0; i < 3; ++i) pos_thr[i] = i + 1 < H ? cb->thr[H + i] : 0.f;
  return true;
}

size_t turbo_rotation_workspace_bytes(int d) { return turbo::rotation_workspace_bytes(d); }

cudaError_t launch_turbo_rotation(uint16_t *Pi, float *Pinv, int d, uint64_t seed, void *ws,
                                  cudaStream_t stream) {
  return turbo::launch_rotation(Pi, Pinv, d, seed, ws, stream);
}

cudaError_t launch_turbo_quantize(const uint16_t *K, int64_t n, int64_t ldk, const uint16_t *Pi,
                                  const uint16_t *S, int m, int d, int bits, uint32_t *codes,
                                  uint16_t *norms, cudaStream_t stream) {
  if (m != d || (d != 64 && d != 128)) return cudaErrorNotSupported;
  const turbo::Codebook *cb = turbo::codebook(d, bits);
#define JL_CASE(TB, DD)                                                                        \
  if (bits == TB && d == DD)                                                                   \
    return turbo::launch_quantize_t<TB, DD>(K, n, ldk, Pi, S, *cb, codes, norms, stream);
  JL_CASE(1, 128) JL_CASE(2, 128) JL_CASE(3, 128) JL_CASE(1, 64) JL_CASE(2, 64) JL_CASE(3, 64)
#undef JL_CASE
  return cudaErrorNotSupported;
}

}  // namespace jlk
