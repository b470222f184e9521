/*
 * jlkey.h -- C ABI of libjlkey: QJL sign-bit compression of attention keys
 * and decode attention that reads only the compressed keys, on NVIDIA B200
 * (sm_100a).
 *
 * The method (cited by page title and section):
 *  - "The Geometry of Forgetting: How Three Papers Cracked KV Cache
 *    Quantization", section "QJL: one bit, zero parameters, unbiased inner
 *    products": a Gaussian sketch S with i.i.d. N(0,1) entries, regenerated
 *    from a seed; the quantizer Q(x) = sign(S x); the dequantizer
 *    Q^-1(z) = sqrt(pi/2)/d * S^T z; the estimator is unbiased (property 1)
 *    with variance shrinking with the number of sketch rows (property 2).
 *  - "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
 *    Overhead", Abstract: quantize one vector (the key) with QJL and apply
 *    the plain JL transform to the other (the query): the asymmetric
 *    estimator.  No per-block zero point or scale is stored.
 *  - same blog page, section "PolarQuant": the radius (norm) that a
 *    direction code drops is stored once per vector in floating point.
 *
 * With m sketch rows (S is m x d) the library computes, per key k:
 *     code(k) = sign(S k)       (m bits, 1 = non-negative)
 *     norm(k) = ||k||_2         (IEEE binary16)
 * and, per query q and key k, the score
 *     s(q,k) = sqrt(pi/2)/m * norm(k) * sum_i (S q)_i * sign(S k)_i
 * which estimates <q,k> (with m = d this is <q, Q^-1(Q(k))> * ||k||).  Decode
 * attention returns  out = sum_t softmax_t(softmax_scale * s(q,k_t)) * v_t.
 *
 * Conventions for every entry point:
 *  - Memory: every buffer is allocated and owned by the caller (device memory
 *    unless stated).  The library allocates nothing, frees nothing and keeps
 *    no pointer after it returns.
 *  - Execution: work is enqueued on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and the call returns without synchronising,
 *    except jl_device_error, which synchronises `stream`.
 *  - Errors: a negative status is returned.  Argument errors are detected
 *    before anything is launched.  JL_ERR_CUDA reports a failed launch.
 *    Kernels never trap; a kernel that detects a fault sets a device error
 *    word that jl_device_error reads and clears.
 *  - Layouts: row-major, innermost index last.  bf16 values are passed as
 *    uint16_t bit patterns, binary16 norms likewise.
 *  - Supported shapes: d in {64, 128}; m in {64, 128, 256, 512}.
 *  - Thread safety: entry points may be called concurrently from several host
 *    threads; the only process-wide state is a per-device cache of device
 *    attributes and addresses, and the test hook of jl_test_drop_copies.
 */
#ifndef JLKEY_H
#define JLKEY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JL_API __attribute__((visibility("default")))
#else
#define JL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream). */
typedef struct CUstream_st *jl_stream_t;

/* Element type of keys and queries. */
typedef enum { JL_BF16 = 0, JL_F32 = 1 } jl_dtype;

enum {
    JL_OK = 0,
    JL_ERR_INVALID_ARG = -1, /* null pointer, negative size, misalignment   */
    JL_ERR_UNSUPPORTED = -2, /* a shape outside the supported set           */
    JL_ERR_WORKSPACE = -3,   /* workspace pointer null or smaller than asked */
    JL_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
    JL_ERR_DEVICE = -5,      /* a kernel reported a fault (jl_device_error) */
    JL_ERR_SCRATCH_LIMIT = -6 /* shapes need more than the static scratch    */
};

/* Human-readable text of a status code (static storage). */
JL_API const char *jl_status_string(int status);

/*
 * jl_sketch_init -- the Gaussian sketch S, regenerated from `seed`.
 * Defines: "The Geometry of Forgetting ...", section "QJL: one bit, zero
 * parameters, unbiased inner products" (S with i.i.d. N(0,1) entries, shared
 * by every vector and rebuilt from a seed).
 *   S    : out, device, m x d bf16, row-major, 16-byte aligned.
 *   Element e = i*d + j is the Box-Muller normal (cosine branch) of the
 *   SplitMix64 outputs 2e and 2e+1 of `seed` (outputs taken from the
 *   generator's counter form: output n = mix(seed + (n+1) * 0x9E3779B97F4A7C15)),
 *   each mapped to the uniform ((x >> 12) + 1/2) * 2^-52, then rounded to
 *   bf16 (nearest, ties to even).
 * Errors: JL_ERR_INVALID_ARG (S null/misaligned), JL_ERR_UNSUPPORTED (m, d).
 */
JL_API int jl_sketch_init(uint16_t *S, int m, int d, uint64_t seed,
                   jl_stream_t stream);

/*
 * jl_quantize_keys -- code(k) and norm(k) for n_keys keys.
 * Defines: same section, quantizer equation Q(x) = sign(S x), plus the norm
 * kept beside the code ("PolarQuant" section: one radius per vector).
 *   K          : in, device, n_keys rows of d elements of `key_dtype`, row r
 *                starting at element r * key_stride; 16-byte aligned base,
 *                key_stride * sizeof(element) a multiple of 16 bytes.
 *   key_dtype  : JL_BF16 (tensor-core path) or JL_F32.
 *   S          : in, device, m x d bf16 from jl_sketch_init (16-byte aligned).
 *   signs      : out, device, n_keys x (m/32) uint32, 16-byte aligned.  Bit i
 *                of the code is bit (i % 32) of word i / 32 (LSB first) and
 *                is 1 iff (S k)_i >= 0.
 *   norms      : out, device, n_keys binary16 (||k||_2 rounded to nearest),
 *                2-byte aligned.
 * n_keys == 0 is a no-op.  Projections are accumulated in fp32 from exact
 * bf16 x bf16 products; a coordinate with |(S k)_i| within the fp32
 * accumulation error of 0 may take either sign.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_CUDA.
 */
JL_API int jl_quantize_keys(const void *K, jl_dtype key_dtype, int64_t n_keys,
                     int64_t key_stride, const uint16_t *S, int m, int d,
                     uint32_t *signs, uint16_t *norms, jl_stream_t stream);

/*
 * jl_quantize_keys_simt -- the same result as jl_quantize_keys computed with
 * plain fp32 FMA on the SIMT cores (no tensor cores).  Serves fp32 keys and
 * cross-checks the tensor-core path.  Same arguments and errors.
 */
JL_API int jl_quantize_keys_simt(const void *K, jl_dtype key_dtype, int64_t n_keys,
                          int64_t key_stride, const uint16_t *S, int m, int d,
                          uint32_t *signs, uint16_t *norms,
                          jl_stream_t stream);

/*
 * jl_decode_workspace_bytes -- device scratch that jl_decode_attention needs
 * for these shapes (query projections and split-context partial softmax
 * states).  Depends on the shapes only.  Returns 0 for unsupported shapes.
 */
JL_API size_t jl_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int m,
                                 int d);

/*
 * jl_decode_attention -- one decode step of attention over compressed keys.
 * Defines: the asymmetric estimator ("QJL ..." Abstract; "The Geometry of
 * Forgetting ...", QJL section, dequantizer equation with m rows, scaled by
 * the stored norm) used as the attention logit, then softmax and the value
 * sum.  Query head h reads KV head h / (Hq / Hkv).
 *   Q        : in, device, B x Hq x d of `q_dtype` (one token per sequence),
 *              16-byte aligned.
 *   S        : in, device, m x d bf16 (the sketch the keys were coded with).
 *   signs    : in, device, B x Hkv x T x (m/32) uint32 codes, 16-byte aligned.
 *   norms    : in, device, B x Hkv x T binary16 key norms, 16-byte aligned.
 *   V        : in, device, B x Hkv x T x d bf16 values, 16-byte aligned.
 *   softmax_scale : logit = softmax_scale * s(q, k_t) (typically 1/sqrt(d)).
 *   out      : out, device, B x Hq x d bf16, 4-byte aligned.
 *   scores   : optional out (NULL to skip), device, B x Hq x T fp32: the
 *              estimator s(q, k_t) before softmax_scale, 4-byte aligned.
 *   workspace: device scratch of at least jl_decode_workspace_bytes(...),
 *              256-byte aligned; contents on entry are ignored.
 * B == 0 is a no-op.  T must be >= 1 (softmax over an empty context is
 * undefined).  Hq must be a multiple of Hkv.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_WORKSPACE,
 * JL_ERR_CUDA.
 */
JL_API int jl_decode_attention(const void *Q, jl_dtype q_dtype, const uint16_t *S,
                        const uint32_t *signs, const uint16_t *norms,
                        const uint16_t *V, int B, int Hq, int Hkv, int64_t T,
                        int m, int d, float softmax_scale, uint16_t *out,
                        float *scores, void *workspace, size_t workspace_bytes,
                        jl_stream_t stream);

/*
 * jl_decode_attention_state -- jl_decode_attention over one part of a context
 * whose keys are spread over several buffers (or GPUs), stopping before the
 * final division: the softmax state of each (b, query head), for
 * jl_merge_attention_states to combine with the other parts' states.
 * Defines: the same estimator, logit and value sum as jl_decode_attention;
 * softmax over a union of disjoint key sets as the log-sum-exp merge of the
 * sets' states (plain algebra of the softmax; the pages do not treat it).
 *   All arguments as jl_decode_attention, for this part's T keys, except:
 *   state    : out, device, B x Hq x (d + 2) fp32, 4-byte aligned (replaces
 *              `out`).  Record (b, h) holds acc[0..d-1], mx, l with
 *              weights w_t = 2^(log2(e) * logit_t - mx): acc = sum_t w_t v_t
 *              and l = sum_t w_t, so the part's output is acc / l.  Only
 *              acc / l and mx + log2(l) are fixed; mx is the kernel's
 *              running maximum.
 *   scores   : optional, B x Hq x T as in jl_decode_attention (this part).
 * Errors: as jl_decode_attention.
 */
JL_API int jl_decode_attention_state(const void *Q, jl_dtype q_dtype, const uint16_t *S,
                              const uint32_t *signs, const uint16_t *norms,
                              const uint16_t *V, int B, int Hq, int Hkv, int64_t T,
                              int m, int d, float softmax_scale, float *state,
                              float *scores, void *workspace, size_t workspace_bytes,
                              jl_stream_t stream);

/*
 * jl_merge_attention_states -- the attention output of a context split into
 * R parts, from the parts' states (jl_decode_attention_state).
 * Defines: softmax over the union of the parts: with M = max over parts of
 * mx_r, out = sum_r 2^(mx_r - M) acc_r / sum_r 2^(mx_r - M) l_r.  A part
 * whose l is 0 (no keys) contributes nothing; a row with no part left is 0.
 *   states   : in, device, R x rows x (d + 2) fp32 (part r's records at
 *              r * rows * (d + 2)), 4-byte aligned.
 *   R        : number of parts, 1 <= R <= 65536.
 *   rows     : records per part (B x Hq), 0 <= rows < 2^31; 0 is a no-op.
 *   d        : 64 or 128.
 *   out      : out, device, rows x d bf16 (nearest), 4-byte aligned.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED (d), JL_ERR_CUDA.
 */
JL_API int jl_merge_attention_states(const float *states, int R, int64_t rows, int d,
                              uint16_t *out, jl_stream_t stream);

/*
 * jl_dequantize_keys -- explicit dequantizer of the codes.
 * Defines: Q^-1(z) = sqrt(pi/2)/d * S^T z ("The Geometry of Forgetting: How
 * Three Papers Cracked KV Cache Quantization", section "QJL: one bit, zero
 * parameters, unbiased inner products"), taken with m sketch rows and with
 * the stored norm restoring the magnitude ("PolarQuant" section):
 *     khat_t = sqrt(pi/2)/m * ||k_t|| * S^T z_t,   z_ti = +1 if bit i is set,
 * so that <q, khat_t> is the asymmetric estimator and E||k - khat||^2 is the
 * page's D_mse, ||k||^2 ((pi/2) d - 1) / m for a Gaussian S.
 *   signs  : in, n_keys x (m/32) uint32 codes (jl_quantize_keys layout),
 *            16-byte aligned.
 *   norms  : in, n_keys binary16 norms.
 *   S      : in, m x d bf16 sketch, 16-byte aligned.
 *   out    : out, n_keys x d bf16 (round to nearest), 16-byte aligned.
 * Computed on the tensor cores with fp32 accumulation.  n_keys == 0 is a
 * no-op.  Errors: JL_ERR_INVALID_ARG (null or misaligned pointer, n_keys < 0),
 * JL_ERR_UNSUPPORTED (m, d), JL_ERR_CUDA.
 */
JL_API int jl_dequantize_keys(const uint32_t *signs, const uint16_t *norms, int64_t n_keys,
                              const uint16_t *S, int m, int d, uint16_t *out,
                              jl_stream_t stream);

/* Largest k of jl_search_topk. */
#define JL_SEARCH_MAX_K 16

/*
 * jl_search_workspace_bytes -- device scratch jl_search_topk needs (query
 * projections of one pass of 128 queries and the per-CTA candidate lists).
 * Depends on the shapes only; 0 for unsupported shapes or k outside
 * [1, JL_SEARCH_MAX_K].
 */
JL_API size_t jl_search_workspace_bytes(int n_queries, int m, int d, int k);

/*
 * jl_search_topk -- inner-product search over a QJL-compressed index.
 * Defines: "The Geometry of Forgetting: How Three Papers Cracked KV Cache
 * Quantization", final section (the quantizer serves any store of vectors
 * read through inner products: vector databases, retrieval), with the
 * asymmetric estimator of the QJL section as the similarity:
 *     s(q, x_j) = sqrt(pi/2)/m * ||x_j|| * <S q, sign(S x_j)>.
 * For every query, the k index vectors with the largest s, best first; equal
 * scores go to the lower index.
 *   Q          : in, n_queries x d of q_dtype (16-byte aligned).
 *   S          : in, m x d bf16 sketch.
 *   signs      : in, n_index x (m/32) uint32 codes (jl_quantize_keys layout),
 *                16-byte aligned.
 *   norms      : in, n_index binary16 norms.
 *   out_index  : out, n_queries x k int32 (-1 past the last vector when
 *                k > n_index).
 *   out_scores : out, n_queries x k fp32 (-inf where out_index is -1).
 *   workspace  : >= jl_search_workspace_bytes(...), 256-byte aligned.
 * Queries are handled 128 at a time.  The scores are computed on the tensor
 * cores with the query projection rounded to fp16 (a power-of-two scale per
 * query keeps its largest coordinate in [2^14, 2^15)), so they agree with the
 * float64 estimator to about 3e-4 of the score scale; near-ties may order
 * differently.  n_queries == 0 is a no-op.  Errors: JL_ERR_INVALID_ARG
 * (n_index < 1, k outside [1, JL_SEARCH_MAX_K], bad pointer), JL_ERR_UNSUPPORTED,
 * JL_ERR_WORKSPACE, JL_ERR_CUDA.
 */
JL_API int jl_search_topk(const void *Q, jl_dtype q_dtype, int n_queries, const uint16_t *S,
                          int m, int d, const uint32_t *signs, const uint16_t *norms,
                          int64_t n_index, int k, int32_t *out_index, float *out_scores,
                          void *workspace, size_t workspace_bytes, jl_stream_t stream);

/*
 * jl_decode_paged_workspace_bytes -- device scratch jl_decode_attention_paged
 * needs (query projections and split partial states) for B sequences of at
 * most max_len keys each (counting the key a call appends).  Depends on the
 * shapes only (the device-side lengths never change it); 0 for unsupported
 * shapes.
 */
JL_API size_t jl_decode_paged_workspace_bytes(int B, int Hq, int Hkv, int64_t max_len,
                                              int m, int d);

/*
 * jl_decode_attention_paged -- one decode step of a batch of sequences of
 * different lengths whose compressed cache lives in a pool of fixed-size
 * pages, optionally appending each sequence's new key first.
 * Defines: the quantizer Q(k) = sign(S k) with the stored norm ("The Geometry
 * of Forgetting ...", QJL and PolarQuant sections) applied to the new key, and
 * the asymmetric estimator of jl_decode_attention used as the attention logit
 * over each sequence's keys.
 *   Q           : in, B x Hq x d of q_dtype (16-byte aligned): the new token's
 *                 queries.
 *   K_new       : in or NULL, B x Hkv x d of k_dtype (16-byte aligned): the new
 *                 token's keys.  When given, key t = seq_lens[b] of sequence b
 *                 is written first: its code and binary16 norm (the
 *                 quantizer of jl_quantize_keys) and its value V_new[b][h]
 *                 go to page block_table[b][t / page_tokens], slot
 *                 t % page_tokens, and the step attends over seq_lens[b] + 1
 *                 keys.  Without K_new it attends over seq_lens[b] keys.
 *   V_new       : in, B x Hkv x d bf16 (required with K_new).
 *   S           : in, m x d bf16 sketch.
 *   sign_pages  : in/out, num_pages x Hkv x page_tokens x (m/32) uint32.
 *   norm_pages  : in/out, num_pages x Hkv x page_tokens binary16.
 *   value_pages : in/out, num_pages x Hkv x page_tokens x d bf16.
 *                 The three pools are 16-byte aligned.
 *   page_tokens : keys per page, a multiple of 32.
 *   block_table : in, B x max_pages int32 page ids (device); entries past a
 *                 sequence's last page are not read.
 *   seq_lens    : in, B int32 (device): keys already cached per sequence.
 *                 Not modified (the caller advances it after an append).
 *                 A length outside [0, max_len] (max_len - 1 with K_new)
 *                 records a device error (jl_device_error) and the
 *                 sequence is clipped to the bound.
 *   max_len     : bound on seq_lens[b] (+1 with K_new), used to size the
 *                 work split and the workspace.
 *   scores      : optional out, B x Hq x max_len fp32 (row stride max_len).
 *   workspace   : >= jl_decode_paged_workspace_bytes(...), 256-byte aligned.
 * A sequence with no key to attend over (seq_lens[b] == 0, no K_new) gets an
 * output of zeros.  Values past a sequence's last key inside its last page
 * are never read into the result, whatever they hold.  The page that
 * receives an appended key must belong to that sequence alone: the other
 * sequences' keys are read while the new keys are being written.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_WORKSPACE,
 * JL_ERR_CUDA.
 */
JL_API int jl_decode_attention_paged(
    const void *Q, jl_dtype q_dtype, const void *K_new, jl_dtype k_dtype,
    const uint16_t *V_new, const uint16_t *S, uint32_t *sign_pages,
    uint16_t *norm_pages, uint16_t *value_pages, int num_pages, int page_tokens,
    const int32_t *block_table, int max_pages, const int32_t *seq_lens, int B, int Hq,
    int Hkv, int64_t max_len, int m, int d, float softmax_scale, uint16_t *out,
    float *scores, void *workspace, size_t workspace_bytes, jl_stream_t stream);

/*
 * jl_decode_attention_noalloc -- jl_decode_attention for callers that cannot
 * allocate device memory.  The paper has no counterpart: this entry point
 * exists for deployment, not for the method.
 * Some callers cannot call cudaMalloc where they call this library: plugins
 * hosted by an engine that owns all device memory through its own pool and
 * gives them no allocator, and code on latency-critical paths where
 * allocating or freeing would stall the device.  This variant takes the same
 * inputs and outputs as jl_decode_attention (same meaning, layout, alignment
 * and errors) but no workspace: its scratch is a statically sized device
 * array inside the library, JL_DECODE_STATIC_SCRATCH_BYTES long, which every
 * GPU that loads the library holds until the process exits.  It allocates
 * and frees nothing.
 *  - Limit: shapes for which jl_decode_workspace_bytes(...) exceeds
 *    JL_DECODE_STATIC_SCRATCH_BYTES are rejected with JL_ERR_SCRATCH_LIMIT
 *    before anything is launched (use jl_decode_attention with a workspace).
 *  - Sharing: every call uses the same array, which keeps the previous call's
 *    contents (no part of it needs to start at zero).  Calls whose kernels
 *    overlap on a GPU, e.g. on two streams, race on it and give wrong
 *    results: serialise them.
 *  - Set-up: the first call made with a given device current looks up the
 *    array's device address on that device; make that first call before any
 *    stream capture.  If that device's context is later destroyed and made
 *    again (cudaDeviceReset), the next call sees the new context and looks
 *    the address up again, so it never launches with a stale one.
 */
#define JL_DECODE_STATIC_SCRATCH_BYTES (16u << 20)
JL_API int jl_decode_attention_noalloc(const void *Q, jl_dtype q_dtype,
                                       const uint16_t *S, const uint32_t *signs,
                                       const uint16_t *norms, const uint16_t *V,
                                       int B, int Hq, int Hkv, int64_t T, int m,
                                       int d, float softmax_scale, uint16_t *out,
                                       float *scores, jl_stream_t stream);

/* ---------------------------------------------------------------------------
 * TurboQuant-prod keys.
 * Defines: "The Geometry of Forgetting: How Three Papers Cracked KV Cache
 * Quantization", sections "Random rotation, and what high dimensions do to
 * your intuitions" (a rotation Pi from an orthogonalised Gaussian matrix; the
 * density f(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2)
 * of each coordinate of a rotated unit vector) and "TurboQuant: bridging MSE
 * and inner product, in two stages" (b-1 bits per coordinate from the
 * Lloyd-Max codebook of f, one more bit from QJL on the residual; unbiased).
 *
 * Per key k (d = 64 or 128; the residual sketch S is m x d with m = d: one
 * residual bit per coordinate):
 *   x = k / ||k||  (0 for k = 0),  y = Pi x  (Pi: the stored bf16 rotation)
 *   cell_i = the cell of the centroid nearest y_i (a value exactly on a
 *            boundary goes to the cell nearer zero; 0 to the cell below it)
 *   r = y - c[cell],  rt = bf16(r)   (nearest, ties to even)
 *   code = cell bit planes, then sign(S rt);  norms = (||k||, ||r||) binary16
 * and per query q, with w = Pi^{-T} q (Pinv from jl_turbo_rotation_init):
 *   s(q, k) = ||k|| * ( <w, c[cell]> + sqrt(pi/2)/m * ||r|| * <S w, sign(S rt)> ).
 * For an exactly orthogonal Pi the QJL stage in this rotated frame is the
 * pages' construction in distribution (S Pi^T is again an i.i.d. Gaussian
 * matrix); mapping the query with the inverse transpose of the stored Pi
 * keeps <w, y> = <q, x> exact, so s is unbiased up to the bf16 rounding of
 * the residual and the binary16 norms.
 *
 * Code layout, per key: words = mse_bits * d/32 + m/32 uint32; plane p
 * (p < mse_bits) is words [p*d/32, (p+1)*d/32) and holds bit p of every
 * coordinate's cell (coordinate i at bit i % 32 of word i / 32 of the
 * plane); the QJL code follows (jl_quantize_keys layout).  norms: n x 2
 * binary16, element 0 = ||k||, element 1 = ||r||.
 * -------------------------------------------------------------------------*/
#define JL_TURBO_MAX_MSE_BITS 3

/*
 * jl_turbo_codebook -- the stage-one codebook: the 2^mse_bits centroids
 * c_0 < ... < c_{L-1} of the Lloyd-Max quantizer of f (centroid = mean of f
 * over its cell, cells bounded by the midpoints of neighbouring centroids),
 * computed in float64 by this library and rounded to float.
 *   centroids : out, HOST memory, 2^mse_bits floats.
 * Errors: JL_ERR_INVALID_ARG (null), JL_ERR_UNSUPPORTED (d < 3, d > 4096,
 * mse_bits outside [1, JL_TURBO_MAX_MSE_BITS]).
 */
JL_API int jl_turbo_codebook(int d, int mse_bits, float *centroids);

/* Device scratch of jl_turbo_rotation_init (0 for unsupported d). */
JL_API size_t jl_turbo_rotation_workspace_bytes(int d);

/*
 * jl_turbo_rotation_init -- the rotation and its query map from `seed`.
 *   Pi   : out, device, d x d bf16, row-major, 16-byte aligned: Q of the
 *          factorisation G = Q R with diag(R) > 0, G[i][j] the normal of
 *          element i*d + j of the jl_sketch_init generator with this seed,
 *          rounded to bf16 (nearest, ties to even).  Orthogonalised in
 *          float64 (Gram-Schmidt with re-orthogonalisation).
 *   Pinv : out, device, d x d fp32, row-major, 16-byte aligned: the inverse
 *          of the bf16 Pi (float64 Newton-Schulz iterations, then rounded).
 *          The decode maps each query as w = Pinv^T q.
 *   workspace : device scratch of jl_turbo_rotation_workspace_bytes(d).
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED (d not 64 or 128),
 * JL_ERR_WORKSPACE, JL_ERR_CUDA.
 */
JL_API int jl_turbo_rotation_init(uint16_t *Pi, float *Pinv, int d, uint64_t seed,
                                  void *workspace, size_t workspace_bytes,
                                  jl_stream_t stream);

/*
 * jl_turbo_quantize_keys -- TurboQuant-prod codes and norms of n_keys keys.
 *   K        : in, device, bf16 keys, row r at element r * key_stride
 *              (16-byte aligned, stride * 2 a multiple of 16 bytes).
 *   Pi       : in, device, d x d bf16 rotation (jl_turbo_rotation_init).
 *   S        : in, device, m x d bf16 residual sketch (jl_sketch_init).
 *   codes    : out, device, n_keys x words uint32 (layout above), 16-byte
 *              aligned.
 *   norms    : out, device, n_keys x 2 binary16, 4-byte aligned.
 * Computed on the tensor cores (both products fp32-accumulated from exact
 * bf16 operands).  A coordinate within the fp32 error of a boundary may take
 * either cell; a residual coordinate within that error of a bf16 rounding
 * midpoint may round either way, and a sign within the resulting error of 0
 * either sign.  n_keys == 0 is a no-op.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED (d, m not equal 64 or 128; key dtype
 * not bf16; mse_bits outside [1, JL_TURBO_MAX_MSE_BITS]), JL_ERR_CUDA.
 */
JL_API int jl_turbo_quantize_keys(const void *K, jl_dtype key_dtype, int64_t n_keys,
                                  int64_t key_stride, const uint16_t *Pi, const uint16_t *S,
                                  int m, int d, int mse_bits, uint32_t *codes,
                                  uint16_t *norms, jl_stream_t stream);

/* Device scratch of jl_turbo_decode_attention (0 for unsupported shapes). */
JL_API size_t jl_turbo_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int m,
                                              int d, int mse_bits);

/*
 * jl_turbo_decode_attention -- one decode step over TurboQuant-prod keys:
 * logit = softmax_scale * s(q, k_t), softmax over the context, value sum.
 * Query head h reads KV head h / (Hq / Hkv).
 *   Q      : in, device, B x Hq x d of `q_dtype`, 16-byte aligned.
 *   Pinv   : in, device, d x d fp32 (jl_turbo_rotation_init).
 *   S      : in, device, m x d bf16 residual sketch.
 *   codes  : in, device, B x Hkv x T x words uint32, 16-byte aligned.
 *   norms  : in, device, B x Hkv x T x 2 binary16, 16-byte aligned.
 *   V      : in, device, B x Hkv x T x d bf16, 16-byte aligned.
 *   out    : out, device, B x Hq x d bf16.
 *   scores : optional out, B x Hq x T fp32 (s before softmax_scale).
 *   workspace : device scratch of jl_turbo_decode_workspace_bytes(...).
 * Supported: d = m = 64 or 128, mse_bits 1 to 3.  B == 0 is a no-op; T >= 1.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_WORKSPACE,
 * JL_ERR_CUDA.
 */
JL_API int jl_turbo_decode_attention(const void *Q, jl_dtype q_dtype, const float *Pinv,
                                     const uint16_t *S, const uint32_t *codes,
                                     const uint16_t *norms, const uint16_t *V, int B, int Hq,
                                     int Hkv, int64_t T, int m, int d, int mse_bits,
                                     float softmax_scale, uint16_t *out, float *scores,
                                     void *workspace, size_t workspace_bytes,
                                     jl_stream_t stream);

/* Device scratch of jl_turbo_decode_attention_paged (0 for unsupported shapes). */
JL_API size_t jl_turbo_decode_paged_workspace_bytes(int B, int Hq, int Hkv, int64_t max_len,
                                                    int m, int d, int mse_bits);

/*
 * jl_turbo_decode_attention_paged -- jl_decode_attention_paged for
 * TurboQuant-prod keys: one decode step of a batch of sequences whose
 * compressed cache lives in a pool of fixed-size pages, optionally appending
 * each sequence's new key first (quantized as by jl_turbo_quantize_keys,
 * with fp32 SIMT products instead of the tensor cores: a coordinate within
 * that rounding of a cell boundary, or a sign within it of 0, may come out
 * either way).  Same page, table, length and error rules as
 * jl_decode_attention_paged; the logit is the TurboQuant-prod score of
 * jl_turbo_decode_attention.
 *   Pi          : in, d x d bf16 rotation (required with K_new).
 *   Pinv        : in, d x d fp32 query map.
 *   S           : in, m x d bf16 residual sketch.
 *   code_pages  : in/out, num_pages x Hkv x page_tokens x ((mse_bits d + m)/32)
 *                 uint32 (the jl_turbo_quantize_keys code layout).
 *   norm_pages  : in/out, num_pages x Hkv x page_tokens x 2 binary16.
 *   value_pages : in/out, num_pages x Hkv x page_tokens x d bf16.
 * Supported: d = m = 64 or 128, mse_bits 1 to 3.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_WORKSPACE,
 * JL_ERR_CUDA.
 */
JL_API int jl_turbo_decode_attention_paged(
    const void *Q, jl_dtype q_dtype, const void *K_new, jl_dtype k_dtype, const uint16_t *V_new,
    const uint16_t *Pi, const float *Pinv, const uint16_t *S, uint32_t *code_pages,
    uint16_t *norm_pages, uint16_t *value_pages, int num_pages, int page_tokens,
    const int32_t *block_table, int max_pages, const int32_t *seq_lens, int B, int Hq, int Hkv,
    int64_t max_len, int m, int d, int mse_bits, float softmax_scale, uint16_t *out,
    float *scores, void *workspace, size_t workspace_bytes, jl_stream_t stream);

/*
 * jl_turbo_dequant_basis -- the reconstruction matrix of the TurboQuant-prod
 * dequantizer, R = [Pi^{-1} | Pi^{-1} S^T] (d x (d + m)), so that
 *     khat = ||k|| * R [ c[cell_0 .. cell_{d-1}] ; sqrt(pi/2)/m ||r|| z ]
 * (jl_turbo_dequantize_keys).  Build it once per (rotation, sketch) pair.
 *   Pinv  : in, device, d x d fp32 query map of jl_turbo_rotation_init
 *           (the inverse of the stored bf16 Pi), 16-byte aligned.
 *   S     : in, device, m x d bf16 residual sketch, 16-byte aligned.
 *   basis : out, device, d x (d + m) binary16, row-major: basis[j][i] =
 *           Pinv[j][i] for i < d, basis[j][d + l] = sum_i Pinv[j][i] S[l][i]
 *           (fp32 products and sums), each rounded to nearest binary16;
 *           16-byte aligned, d (d + m) elements.
 * Supported: d = m = 64 or 128.
 * Errors: JL_ERR_INVALID_ARG (null or misaligned pointer), JL_ERR_UNSUPPORTED
 * (d, m), JL_ERR_CUDA.
 */
JL_API int jl_turbo_dequant_basis(const float *Pinv, const uint16_t *S, int m, int d,
                                  uint16_t *basis, jl_stream_t stream);

/*
 * jl_turbo_dequantize_keys -- explicit TurboQuant-prod dequantizer Q_prod^-1.
 * Defines: "The Geometry of Forgetting: How Three Papers Cracked KV Cache
 * Quantization", section "TurboQuant: bridging MSE and inner product, in two
 * stages" (the QJL estimate of the residual added back to the stage-one
 * reconstruction), in the rotated frame, mapped back with the inverse of the
 * stored rotation and scaled by the key norm:
 *     khat_t = ||k_t|| * Pi^{-1} ( c[cell_t] + sqrt(pi/2)/m ||r_t|| S^T z_t ),
 * z_ti = +1 if residual bit i is set, so <q, khat_t> is the TurboQuant-prod
 * estimate s(q, k_t) of jl_turbo_decode_attention.  Computed as
 * ||k_t|| * basis a_t on the tensor cores (binary16 operands, fp32
 * accumulation) with a_t = [ binary16(c[cell_ti]) ; binary16(sqrt(pi/2)/m
 * ||r_t||) z_t ] (the centroids of jl_turbo_codebook rounded to binary16;
 * ||r_t|| the stored binary16 norm, the product in fp32 then rounded).
 *   codes : in, device, n_keys x ((mse_bits d + m)/32) uint32
 *           (jl_turbo_quantize_keys layout), 16-byte aligned.
 *   norms : in, device, n_keys x 2 binary16 (||k||, ||r||), 4-byte aligned.
 *   basis : in, device, d x (d + m) binary16 from jl_turbo_dequant_basis,
 *           16-byte aligned.
 *   out   : out, device, n_keys x d bf16 (round to nearest), 16-byte aligned.
 * Supported: d = m = 64 or 128, mse_bits 1 to JL_TURBO_MAX_MSE_BITS.  n_keys == 0
 * is a no-op.
 * Errors: JL_ERR_INVALID_ARG (null or misaligned pointer, n_keys < 0),
 * JL_ERR_UNSUPPORTED (d, m, mse_bits, n_keys >= 2^40), JL_ERR_CUDA.
 */
JL_API int jl_turbo_dequantize_keys(const uint32_t *codes, const uint16_t *norms,
                                    int64_t n_keys, const uint16_t *basis, int m, int d,
                                    int mse_bits, uint16_t *out, jl_stream_t stream);

/*
 * jl_device_error -- synchronise `stream`, then read and clear the device
 * error word of the current device (0 = no fault reported).  *code receives
 * the word.  Returns JL_OK, JL_ERR_DEVICE when the word was non-zero, or
 * JL_ERR_CUDA.  Codes: JL_DERR_TC_WAIT_TIMEOUT (a tensor-core kernel's
 * pipeline wait ran out), JL_DERR_DECODE_PLAN (a decode work split or a
 * paged length did not fit), JL_DERR_DECODE_WAIT_TIMEOUT (a decode copy wait
 * ran out), JL_DERR_INDEX (see below).
 */
enum {
    JL_DERR_TC_WAIT_TIMEOUT = 1,
    JL_DERR_DECODE_PLAN = 3,
    JL_DERR_DECODE_WAIT_TIMEOUT = 4,
    JL_DERR_INDEX = 5 /* index-checking debug build only: a kernel computed an
                         index outside the extent the call's shapes give a
                         buffer, and skipped that access */
};
JL_API int jl_device_error(int *code, jl_stream_t stream);

/*
 * jl_test_drop_copies -- failure detection test hook (not part of the
 * method; for tests only).  Every wait inside the library's kernels is
 * bounded; when one runs out the kernel records a code in the device error
 * word, lets the copies it started land, frees its tensor memory and returns,
 * leaving the context usable.  To exercise that path without any GPU fault,
 * enable = 1 makes the launches that follow of the tensor-core quantizer
 * (jl_quantize_keys, bf16 keys) and of the contiguous decode scorer
 * (jl_decode_attention, jl_decode_attention_noalloc) start no copy at all,
 * so their waits run out; their outputs are then undefined.  wait_limit_ns
 * (1e3 .. 2e9, 0 = the default 2e9) bounds, in GPU time, every wait of those
 * two kernels launched after the call.  enable = 0 with wait_limit_ns = 0
 * restores normal operation.  Process-wide; calls made while it is on from
 * other threads are affected too.  Returns JL_OK or JL_ERR_INVALID_ARG.
 */
JL_API int jl_test_drop_copies(int enable, uint64_t wait_limit_ns);

/*
 * jl_build_flags -- how this copy of the library was built (not part of the
 * method): a bit set of JL_BUILD_* flags.  JL_BUILD_INDEX_CHECKS: the
 * index-checking debug build, whose kernels check every global access they
 * make through a raw pointer against the extent the call's shapes give that
 * buffer, skip one that falls outside and report JL_DERR_INDEX.
 */
enum { JL_BUILD_INDEX_CHECKS = 1 };
JL_API int jl_build_flags(void);

/*
 * jl_bf16_from_f64 -- host helper: the bf16 code (round to nearest, ties to
 * even, directly from float64) that jl_sketch_init applies to each normal.
 */
JL_API uint16_t jl_bf16_from_f64(double x);

#ifdef __cplusplus
}
#endif

#endif /* JLKEY_H */
