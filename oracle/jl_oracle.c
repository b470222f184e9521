/*
 * jl_oracle.c -- plain, slow, float64 CPU oracle for QJL sign-bit key
 * compression and compressed-key decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library in bit_jl_key_b200/.
 *
 * Sources (cited by page title and section):
 *  [QJL-abs]  "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization
 *             with Zero Overhead", Abstract: a JL transform followed by
 *             sign-bit quantization; the asymmetric estimator quantizes one
 *             vector and applies the plain JL transform to the other.
 *  [GEO-QJL]  "The Geometry of Forgetting: How Three Papers Cracked KV Cache
 *             Quantization", section "QJL: one bit, zero parameters, unbiased
 *             inner products": S has i.i.d. N(0,1) entries and is regenerated
 *             from a seed; quantizer Q(x) = sign(S x); dequantizer
 *             Q^-1(z) = sqrt(pi/2)/d * S^T z; properties 1 (unbiased) and
 *             2 (variance); attention logits are exactly such inner
 *             products, which is why the estimator serves attention.
 *  [GEO-POLAR] same page, section "PolarQuant": the radius (norm) is kept
 *             separately in floating point, one number per vector.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - S is m x d (m sketch rows), the rescale is sqrt(pi/2)/m; with m = d this
 *    is exactly the dequantizer equation of [GEO-QJL].
 *  - The magnitude lost by the sign step is restored by the stored key norm:
 *    <q,k> ~= sqrt(pi/2)/m * ||k|| * <S q, sign(S k)>.
 *  - sign(0) = +1.  Bit i of the code is 1 iff (S k)_i >= 0; bits are packed
 *    LSB-first into 32-bit words, word w holding rows 32w .. 32w+31.
 *  - S is drawn with SplitMix64 (Steele, Lea & Flood, "Fast splittable
 *    pseudorandom number generators", OOPSLA 2014) used as a counter-based
 *    generator, turned into normals by the Box-Muller transform (cosine
 *    branch), and rounded to bfloat16 (round to nearest, ties to even).
 *    Element e = i*d + j of S uses generator outputs 2e and 2e+1.
 *  - Decode attention: logits = softmax_scale * score, softmax over the
 *    context, output = sum_t p_t v_t.  Query head h reads KV head
 *    h / (Hq/Hkv) (grouped-query attention).
 *
 * Everything is computed in float64 in the order the definitions state; a
 * library call (sqrt, log, cos, exp) is used as a step where one is named.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define JLO_PI 3.14159265358979323846264338327950288

/* ---------------------------------------------------------------------- */
/* SplitMix64 (Steele, Lea & Flood 2014).  The sequential generator keeps a
 * 64-bit state, adds the odd constant gamma = 0x9E3779B97F4A7C15 on every
 * call, and returns a mixed copy of the new state.  Because the state after
 * n+1 calls is seed + (n+1)*gamma, the n-th output (0-based) can be computed
 * directly: this is the counter-based form used here. */
static uint64_t jlo_sm64_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t jlo_splitmix64(uint64_t seed, uint64_t n)
{
    uint64_t state = seed + (n + 1ULL) * 0x9E3779B97F4A7C15ULL;
    return jlo_sm64_mix(state);
}

/* Uniform in the open interval (0,1): the top 52 bits, offset by half a step
 * (j + 1/2) * 2^-52, so the result is never 0 (log() below stays finite) and
 * never rounds up to 1 (j + 1/2 < 2^52 needs only 53 significant bits). */
double jlo_uniform(uint64_t bits)
{
    return ((double)(bits >> 12) + 0.5) * (1.0 / 4503599627370496.0);
}

/* Standard normal for element e of the sketch (Box-Muller, cosine branch). */
double jlo_gauss(uint64_t seed, uint64_t e)
{
    double u1 = jlo_uniform(jlo_splitmix64(seed, 2ULL * e));
    double u2 = jlo_uniform(jlo_splitmix64(seed, 2ULL * e + 1ULL));
    return sqrt(-2.0 * log(u1)) * cos(2.0 * JLO_PI * u2);
}

/* ---------------------------------------------------------------------- */
/* float64 -> bfloat16, round to nearest, ties to even.  Done on values:
 * x = f * 2^e with f in [0.5,1); a bfloat16 carries 8 significant bits, so
 * the rounded value is nearbyint(f * 2^8) * 2^(e-8) (nearbyint rounds ties to
 * even in the default rounding mode).  Values below the smallest normal use
 * the fixed subnormal step 2^-133.  The rounded value is exactly a bfloat16,
 * so its float32 bit pattern's top half is the code. */
uint16_t jlo_f64_to_bf16(double x)
{
    union { float f; uint32_t u; } cv;
    if (isnan(x)) return 0x7FC0;
    double ax = fabs(x);
    double r;
    if (ax == 0.0) {
        r = 0.0;
    } else if (ax < ldexp(1.0, -126)) {
        r = nearbyint(ldexp(ax, 133)) * ldexp(1.0, -133);
    } else {
        int e;
        double f = frexp(ax, &e);
        r = ldexp(nearbyint(ldexp(f, 8)), e - 8);
    }
    /* largest finite bfloat16 is (2 - 2^-7) * 2^127 */
    if (r > ldexp(2.0 - ldexp(1.0, -7), 127)) r = INFINITY;
    cv.f = (float)r;          /* exact: r is a bfloat16 value (or inf) */
    uint16_t code = (uint16_t)(cv.u >> 16);
    if (signbit(x)) code |= 0x8000;
    return code;
}

void jlo_f64_to_bf16_array(long n, const double *x, uint16_t *out)
{
    for (long i = 0; i < n; ++i) out[i] = jlo_f64_to_bf16(x[i]);
}

double jlo_bf16_to_f64(uint16_t code)
{
    union { float f; uint32_t u; } cv;
    cv.u = ((uint32_t)code) << 16;
    return (double)cv.f;
}

/* ---------------------------------------------------------------------- */
/* Sketch S[i][j], i < m, j < d: the bfloat16 code of the normal drawn for
 * element e = i*d + j.  [GEO-QJL]: one S serves every vector and is rebuilt
 * from its seed rather than stored. */
void jlo_sketch_bf16(int m, int d, uint64_t seed, uint16_t *S_bits)
{
    long total = (long)m * d;
    #pragma omp parallel for schedule(static)
    for (long e = 0; e < total; ++e)
        S_bits[e] = jlo_f64_to_bf16(jlo_gauss(seed, (uint64_t)e));
}

/* ---------------------------------------------------------------------- */
/* Quantizer [GEO-QJL] Q(x) = sign(S x), one bit per sketch row, plus the key
 * norm that the sign step discards [GEO-POLAR].
 *   K      : n x d keys (values as stored, widened to float64), row stride ldk
 *   S      : m x d sketch (float64), row-major
 *   signs  : n x (m/32) words, LSB-first
 *   norms  : n exact norms ||k||_2 (float64; storage rounding is the caller's)
 *   band   : optional n x m flags, 1 where |(S k)_i| < band_rel * ||k||
 */
void jlo_quantize(long n, int d, int m, const double *K, long ldk,
                  const double *S, uint32_t *signs, double *norms,
                  double band_rel, uint8_t *band)
{
    int words = m / 32;
    #pragma omp parallel for schedule(static)
    for (long t = 0; t < n; ++t) {
        const double *k = K + t * ldk;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += k[j] * k[j];
        double nk = sqrt(ss);
        norms[t] = nk;
        for (int w = 0; w < words; ++w) signs[t * words + w] = 0u;
        for (int i = 0; i < m; ++i) {
            double y = 0.0;
            for (int j = 0; j < d; ++j) y += S[(long)i * d + j] * k[j];
            if (y >= 0.0) signs[t * words + i / 32] |= (1u << (i % 32));
            if (band) band[t * m + i] = (fabs(y) < band_rel * nk) ? 1 : 0;
        }
    }
}

/* Plain JL transform of the query side [QJL-abs]: u = S q. */
void jlo_project(long n, int d, int m, const double *Q, const double *S,
                 double *U)
{
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < n; ++r)
        for (int i = 0; i < m; ++i) {
            double y = 0.0;
            for (int j = 0; j < d; ++j) y += S[(long)i * d + j] * Q[r * d + j];
            U[r * m + i] = y;
        }
}

/* Asymmetric estimator [GEO-QJL] with m rows:
 *   <q,k> ~= <q, Q^-1(Q(k))> scaled by ||k||
 *          = sqrt(pi/2)/m * ||k|| * sum_i (S q)_i * sign(S k)_i
 * u = S q (m values), one code and one norm per key. */
double jlo_estimate_one(int m, const double *u, const uint32_t *code,
                        double norm)
{
    double acc = 0.0;
    for (int i = 0; i < m; ++i) {
        double sigma = ((code[i / 32] >> (i % 32)) & 1u) ? 1.0 : -1.0;
        acc += u[i] * sigma;
    }
    return sqrt(JLO_PI / 2.0) / (double)m * norm * acc;
}

void jlo_scores(long T, int m, const double *u, const uint32_t *signs,
                const double *norms, double *out)
{
    int words = m / 32;
    #pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t)
        out[t] = jlo_estimate_one(m, u, signs + t * words, norms[t]);
}

/* Dequantizer [GEO-QJL] Q^-1(z) = sqrt(pi/2)/d * S^T z, taken with m sketch
 * rows and with the stored norm restoring the magnitude [GEO-POLAR]:
 *   khat = sqrt(pi/2)/m * ||k|| * S^T z,   z_i = +1 if bit i is set, else -1
 *   signs : n x (m/32) words, LSB-first
 *   norms : n norms (float64 values of the stored norms)
 *   S     : m x d (float64), row-major
 *   out   : n x d reconstructions */
void jlo_dequantize(long n, int d, int m, const uint32_t *signs,
                    const double *norms, const double *S, double *out)
{
    int words = m / 32;
    #pragma omp parallel for schedule(static)
    for (long t = 0; t < n; ++t) {
        const uint32_t *code = signs + t * words;
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int i = 0; i < m; ++i) {
                double z = ((code[i / 32] >> (i % 32)) & 1u) ? 1.0 : -1.0;
                acc += S[(long)i * d + j] * z;
            }
            out[t * d + j] = sqrt(JLO_PI / 2.0) / (double)m * norms[t] * acc;
        }
    }
}

/* ---------------------------------------------------------------------- */
/* Decode attention over compressed keys: the attention logits are the inner
 * products that the estimator of [GEO-QJL] approximates.  One query token per
 * (b, hq).
 *   Q      : B x Hq x d           (float64 values of the stored query)
 *   S      : m x d
 *   signs  : B x Hkv x T x (m/32)
 *   norms  : B x Hkv x T          (float64 values of the stored norms)
 *   V      : B x Hkv x T x d      (float64 values of the stored values)
 *   out    : B x Hq x d
 *   scores : optional B x Hq x T, the estimator before softmax_scale
 * Softmax is taken with its maximum subtracted, in float64. */
void jlo_decode(int B, int Hq, int Hkv, long T, int m, int d,
                const double *Q, const double *S, const uint32_t *signs,
                const double *norms, const double *V, double softmax_scale,
                double *out, double *scores)
{
    int G = Hq / Hkv;
    int words = m / 32;
    #pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < B * Hq; ++bh) {
        int b = bh / Hq, h = bh % Hq, hk = h / G;
        const double *q = Q + (long)bh * d;
        double u[4096];
        for (int i = 0; i < m; ++i) {
            double y = 0.0;
            for (int j = 0; j < d; ++j) y += S[(long)i * d + j] * q[j];
            u[i] = y;
        }
        long base = ((long)b * Hkv + hk) * T;
        /* pass 1: scores and their maximum */
        double mx = -INFINITY;
        for (long t = 0; t < T; ++t) {
            double s = jlo_estimate_one(m, u, signs + (base + t) * words,
                                        norms[base + t]);
            if (scores) scores[(long)bh * T + t] = s;
            double l = s * softmax_scale;
            if (l > mx) mx = l;
        }
        /* pass 2: softmax weights and the value sum */
        double den = 0.0;
        double *o = out + (long)bh * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (long t = 0; t < T; ++t) {
            double s = jlo_estimate_one(m, u, signs + (base + t) * words,
                                        norms[base + t]);
            double p = exp(s * softmax_scale - mx);
            den += p;
            const double *v = V + (base + t) * d;
            for (int j = 0; j < d; ++j) o[j] += p * v[j];
        }
        for (int j = 0; j < d; ++j) o[j] /= den;
    }
}

/* Exact attention with the unquantized keys (context only; never a parity
 * criterion).  Same layouts as jlo_decode with K (B x Hkv x T x d). */
void jlo_exact_attention(int B, int Hq, int Hkv, long T, int d,
                         const double *Q, const double *K, const double *V,
                         double softmax_scale, double *out, double *scores)
{
    int G = Hq / Hkv;
    #pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < B * Hq; ++bh) {
        int b = bh / Hq, h = bh % Hq, hk = h / G;
        const double *q = Q + (long)bh * d;
        long base = ((long)b * Hkv + hk) * T;
        double mx = -INFINITY;
        for (long t = 0; t < T; ++t) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += q[j] * K[(base + t) * d + j];
            if (scores) scores[(long)bh * T + t] = s;
            if (s * softmax_scale > mx) mx = s * softmax_scale;
        }
        double den = 0.0;
        double *o = out + (long)bh * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (long t = 0; t < T; ++t) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += q[j] * K[(base + t) * d + j];
            double p = exp(s * softmax_scale - mx);
            den += p;
            for (int j = 0; j < d; ++j) o[j] += p * V[(base + t) * d + j];
        }
        for (int j = 0; j < d; ++j) o[j] /= den;
    }
}

/* ---------------------------------------------------------------------- */
/* Storage overhead of a block quantizer ("The overhead nobody tells you
 * about", same page): b bits per number plus a zero point and a scale of
 * const_bits in total, shared by a block of `block` numbers. */
double jlo_block_effective_bits(double b, double block, double const_bits)
{
    return b + const_bits / block;
}

/* Bits a QJL-compressed key occupies per coordinate of the original key:
 * m sign bits plus one stored norm of norm_bits, spread over d coordinates. */
double jlo_qjl_bits_per_coordinate(int m, int d, int norm_bits)
{
    return ((double)m + (double)norm_bits) / (double)d;
}

int jlo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
