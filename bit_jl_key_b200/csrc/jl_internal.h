// jl_internal.h -- launchers behind the C ABI (host side, internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "jlkey.h"

namespace jlk {

cudaError_t launch_sketch(uint16_t *S, int m, int d, uint64_t seed,
                          cudaStream_t stream);

// SIMT quantizer: any supported (m, d), bf16 or fp32 keys.
cudaError_t launch_quantize_simt(const void *K, bool keys_f32, int64_t n,
                                 int64_t ldk, const uint16_t *S, int m, int d,
                                 uint32_t *signs, uint16_t *norms,
                                 cudaStream_t stream);

// Tensor-core (tcgen05 + TMA) quantizer for bf16 keys.  Returns
// cudaErrorNotSupported when the shape is outside its envelope, in which case
// the caller falls back to the SIMT path.
cudaError_t launch_quantize_tc(const uint16_t *K, int64_t n, int64_t ldk,
                               const uint16_t *S, int m, int d,
                               uint32_t *signs, uint16_t *norms,
                               cudaStream_t stream);
bool quantize_tc_supported(int m, int d, int64_t n, int64_t ldk, const void *K);

// Tensor-core dequantizer khat = sqrt(pi/2)/m * ||k|| * S^T z (bf16 out).
cudaError_t launch_dequantize_tc(const uint32_t *signs, const uint16_t *norms, int64_t n,
                                 const uint16_t *S, int m, int d, uint16_t *out,
                                 cudaStream_t stream);

// TurboQuant-prod dequantizer (dequant_tc.cu): the reconstruction matrix
// R = [Pinv | Pinv S^T] in binary16 (d x (d + m)), and khat = ||k|| R a on
// the tensor cores (d = m = 128).
cudaError_t launch_turbo_dequant_basis(const float *Pinv, const uint16_t *S, int m, int d,
                                       uint16_t *basis, cudaStream_t stream);
cudaError_t launch_turbo_dequantize(const uint32_t *codes, const uint16_t *norms, int64_t n,
                                    const uint16_t *basis, int m, int d, int bits,
                                    uint16_t *out, cudaStream_t stream);

// u = S q for nq queries (fp32 [nq][m]).
cudaError_t launch_query_projection(const void *Q, bool q_f32, const uint16_t *S, float *U,
                                    int nq, int m, int d, cudaStream_t stream);

// Inner-product top-k search over a compressed index (search_tc.cu).
size_t search_workspace_bytes(int nq, int m, int k);
cudaError_t launch_search(const void *Q, bool q_f32, int nq, const uint16_t *S, int m, int d,
                          const uint32_t *signs, const uint16_t *norms, int64_t N, int k,
                          int32_t *out_idx, float *out_scores, void *workspace,
                          cudaStream_t stream);

// 2-D bf16 tensor map [rows][cols] (pitch in elements), boxes of 64 columns x
// box_rows rows, 128-byte swizzle (quantize_tc.cu).
namespace tc {
bool make_map(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols,
              uint64_t pitch_elems, uint32_t box_rows);
}

// TurboQuant-prod (turbo_tc.cu): the stage-one codebook (host, cached; false
// for unsupported d / bits), its odd Walsh coefficients (walsh[4]), the rotation
// and its inverse, and the tensor-core quantizer (d = m = 128, bf16 keys).
bool turbo_codebook(int d, int bits, float *centroids, double *walsh);
size_t turbo_rotation_workspace_bytes(int d);
cudaError_t launch_turbo_rotation(uint16_t *Pi, float *Pinv, int d, uint64_t seed, void *ws,
                                  cudaStream_t stream);
cudaError_t launch_turbo_quantize(const uint16_t *K, int64_t n, int64_t ldk, const uint16_t *Pi,
                                  const uint16_t *S, int m, int d, int bits, uint32_t *codes,
                                  uint16_t *norms, cudaStream_t stream);

// Decode: work split shared by the workspace query and the launch.
struct DecodePlan {
  int B, Hq, Hkv, m, d;
  int64_t T;     // keys per unit (contiguous cache) or the bound max_len (paged)
  int G;         // query heads per KV head
  int HG;        // head groups per KV head (groups of at most 8 heads)
  int units;     // B * Hkv * HG
  int64_t nb_u;  // 32-key blocks per unit (paged: the bound)
  int64_t NB;    // units * nb_u (paged: the bound)
  int W;         // bound on the warps launched
  int records;   // partial-state records: W + units
  size_t u_bytes;        // fp32 query projections [B][Hq][m]
  size_t partial_bytes;  // fp32 [records][8][d + 2]
  size_t total_bytes;
};
bool make_decode_plan(int B, int Hq, int Hkv, int64_t T, int m, int d,
                      DecodePlan *plan);
bool make_paged_plan(int B, int Hq, int Hkv, int64_t max_len, int m, int d,
                     DecodePlan *plan);

// TurboQuant-prod decode (decode.cu): d = m = 128, bits 1 to 3.
bool make_turbo_decode_plan(int B, int Hq, int Hkv, int64_t T, int m, int d, int bits,
                            DecodePlan *plan);
cudaError_t launch_turbo_decode(const DecodePlan &pl, int bits, const void *Q, bool q_f32,
                                const float *Pinv, const uint16_t *S, const uint32_t *codes,
                                const uint16_t *norms, const uint16_t *V, const double *walsh,
                                float softmax_scale, uint16_t *out, float *scores,
                                void *workspace, cudaStream_t stream);

// Argument checks of jl_decode_attention that do not involve the workspace
// (dtype, shapes, null pointers, alignment) and the work split they imply.
// Returns JL_OK with *plan filled, or the status the entry point returns.
// *empty is set when B == 0 (nothing to do).
int validate_decode(const void *Q, jl_dtype q_dtype, const uint16_t *S,
                    const uint32_t *signs, const uint16_t *norms, const uint16_t *V,
                    int B, int Hq, int Hkv, int64_t T, int m, int d, float softmax_scale,
                    const uint16_t *out, const float *scores, DecodePlan *plan,
                    bool *empty);

cudaError_t launch_decode(const DecodePlan &p, const void *Q, bool q_f32,
                          const uint16_t *S, const uint32_t *signs,
                          const uint16_t *norms, const uint16_t *V,
                          float softmax_scale, uint16_t *out, float *scores,
                          void *workspace, cudaStream_t stream, float *state = nullptr);

// Merge R attention states per row ([R][rows][d + 2], each (acc, max, sum))
// into bf16 rows [rows][d].
cudaError_t launch_merge_states(const float *states, int R, int64_t rows, int d,
                                uint16_t *out, cudaStream_t stream);

struct PagedArgs {
  const void *Q;
  bool q_f32;
  const void *K_new;  // nullable: no append
  bool k_f32;
  const uint16_t *V_new;
  const uint16_t *S;
  uint32_t *sign_pages;
  uint16_t *norm_pages;
  uint16_t *value_pages;
  int num_pages, page_tokens;
  const int32_t *block_table;
  int max_pages;
  const int32_t *seq_lens;
  float softmax_scale;
  uint16_t *out;
  float *scores;
  void *workspace;
};
cudaError_t launch_decode_paged(const DecodePlan &p, const PagedArgs &a,
                                cudaStream_t stream);

// TurboQuant-prod paged step (decode.cu): PagedArgs with sign_pages holding
// the full codes ((bits d + m)/32 words per key) and norm_pages the binary16
// (||k||, ||r||) pairs, plus the rotation, its query map and the codebook.
struct TurboPagedArgs {
  const uint16_t *Pi;
  const float *Pinv;
  double walsh[4];
  float mag[4];      // centroid magnitudes, positive half
  float pos_thr[3];  // positive boundaries between them
};
cudaError_t launch_turbo_decode_paged(const DecodePlan &p, int bits, const PagedArgs &a,
                                      const TurboPagedArgs &t, cudaStream_t stream);
// The codebook's centroid magnitudes and positive boundaries (float).
bool turbo_magnitudes(int d, int bits, float *mag, float *pos_thr);

}  // namespace jlk
