// api.cu -- the extern "C" entry points of libjlkey (include/jlkey.h).
//
// Every entry point validates its arguments on the host before launching
// anything and returns a status code; no exception crosses the boundary.
#include "jl_common.cuh"
#include "jl_internal.h"

#include <atomic>
#include <mutex>

namespace jlk {

__device__ int g_device_error = 0;

namespace {
std::atomic<int> g_drop_copies{0};
std::atomic<unsigned long long> g_wait_limit_ns{WAIT_LIMIT_NS};
}  // namespace

bool test_drop_copies() { return g_drop_copies.load(std::memory_order_relaxed) != 0; }
unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_attr_mu;
int g_sm_count[kMaxDevices];
int g_smem_optin[kMaxDevices];
int *g_err_ptr[kMaxDevices];
unsigned long long g_err_ctx[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev;
}
}  // namespace

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (g_sm_count[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess || v <= 0)
      v = 148;
    g_sm_count[dev] = v;
  }
  return g_sm_count[dev];
}

int *device_error_ptr() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (g_err_ptr[dev] == nullptr || g_err_ctx[dev] != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int *>(p);
    g_err_ctx[dev] = ctx;
  }
  return g_err_ptr[dev];
}

unsigned long long current_context_id() {
  using GetCurrent = int (*)(void **);
  using GetId = int (*)(void *, unsigned long long *);
  static std::once_flag once;
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  std::call_once(once, [] {
    void *a = nullptr, *b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) ==
            cudaSuccess && qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrent>(a);
      get_id = reinterpret_cast<GetId>(b);
    }
  });
  if (!get_current || !get_id) return 0;
  // 0 also when no context is bound to this thread yet: the first lookup made
  // under id 0 is then repeated once the runtime has bound one
  void *ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != 0 || ctx == nullptr || get_id(ctx, &id) != 0) return 0;
  return id;
}

void *tensor_map_encoder() {
  static std::once_flag once;
  static void *fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  });
  return fn;
}

int device_max_smem_optin() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 227 * 1024;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (g_smem_optin[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               dev) != cudaSuccess || v <= 0)
      v = 227 * 1024;
    g_smem_optin[dev] = v;
  }
  return g_smem_optin[dev];
}

int validate_decode(const void *Q, jl_dtype q_dtype, const uint16_t *S,
                    const uint32_t *signs, const uint16_t *norms, const uint16_t *V,
                    int B, int Hq, int Hkv, int64_t T, int m, int d, float softmax_scale,
                    const uint16_t *out, const float *scores, DecodePlan *plan,
                    bool *empty) {
  auto al = [](const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
  };
  *empty = false;
  if (q_dtype != JL_BF16 && q_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv != 0) return JL_ERR_INVALID_ARG;
  if (!((d == 64 || d == 128) && (m == 64 || m == 128 || m == 256 || m == 512)))
    return JL_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale)) return JL_ERR_INVALID_ARG;  // NaN
  if (B == 0) {
    *empty = true;
    return JL_OK;
  }
  if (!Q || !S || !signs || !norms || !V || !out) return JL_ERR_INVALID_ARG;
  if (!al(Q, 16) || !al(S, 16) || !al(signs, 16) || !al(norms, 16) || !al(V, 16) ||
      !al(out, 4) || (scores && !al(scores, 4)))
    return JL_ERR_INVALID_ARG;
  if (!make_decode_plan(B, Hq, Hkv, T, m, d, plan)) return JL_ERR_UNSUPPORTED;
  return JL_OK;
}

}  // namespace jlk

namespace {

bool aligned(const void *p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

bool supported_md(int m, int d) {
  return (d == 64 || d == 128) && (m == 64 || m == 128 || m == 256 || m == 512);
}

// TurboQuant-prod shapes: one residual bit per coordinate, m = d = 64 or 128
static bool turbo_md(int m, int d) { return m == d && (d == 64 || d == 128); }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? JL_OK : JL_ERR_CUDA; }

int validate_quantize(const void *K, jl_dtype kt, int64_t n, int64_t ldk,
                      const uint16_t *S, int m, int d, const uint32_t *signs,
                      const uint16_t *norms) {
  if (kt != JL_BF16 && kt != JL_F32) return JL_ERR_INVALID_ARG;
  if (n < 0) return JL_ERR_INVALID_ARG;
  if (!supported_md(m, d)) return JL_ERR_UNSUPPORTED;
  if (n == 0) return JL_OK;
  if (!K || !S || !signs || !norms) return JL_ERR_INVALID_ARG;
  if (ldk < d) return JL_ERR_INVALID_ARG;
  const size_t esz = (kt == JL_F32) ? 4 : 2;
  if (!aligned(K, 16) || ((size_t)ldk * esz) % 16 != 0) return JL_ERR_INVALID_ARG;
  if (!aligned(S, 16) || !aligned(signs, 16) || !aligned(norms, 2))
    return JL_ERR_INVALID_ARG;
  return JL_OK;
}

}  // namespace

extern "C" {

const char *jl_status_string(int status) {
  switch (status) {
    case JL_OK: return "ok";
    case JL_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or misaligned buffer)";
    case JL_ERR_UNSUPPORTED: return "unsupported shape (d must be 64 or 128, m one of 64/128/256/512)";
    case JL_ERR_WORKSPACE: return "workspace missing or smaller than jl_decode_workspace_bytes()";
    case JL_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case JL_ERR_DEVICE: return "a kernel reported a device-side fault";
    case JL_ERR_SCRATCH_LIMIT: return "shapes need more scratch than the static decode scratch (JL_DECODE_STATIC_SCRATCH_BYTES); use jl_decode_attention with a workspace";
    default: return "unknown status";
  }
}

int jl_sketch_init(uint16_t *S, int m, int d, uint64_t seed,
                   jl_stream_t stream) {
  if (!supported_md(m, d)) return JL_ERR_UNSUPPORTED;
  if (!S || !aligned(S, 16)) return JL_ERR_INVALID_ARG;
  return from_cuda(jlk::launch_sketch(S, m, d, seed, (cudaStream_t)stream));
}

int jl_quantize_keys_simt(const void *K, jl_dtype key_dtype, int64_t n_keys,
                          int64_t key_stride, const uint16_t *S, int m, int d,
                          uint32_t *signs, uint16_t *norms,
                          jl_stream_t stream) {
  int st = validate_quantize(K, key_dtype, n_keys, key_stride, S, m, d, signs,
                             norms);
  if (st != JL_OK || n_keys == 0) return st;
  return from_cuda(jlk::launch_quantize_simt(K, key_dtype == JL_F32, n_keys,
                                             key_stride, S, m, d, signs, norms,
                                             (cudaStream_t)stream));
}

int jl_quantize_keys(const void *K, jl_dtype key_dtype, int64_t n_keys,
                     int64_t key_stride, const uint16_t *S, int m, int d,
                     uint32_t *signs, uint16_t *norms, jl_stream_t stream) {
  int st = validate_quantize(K, key_dtype, n_keys, key_stride, S, m, d, signs,
                             norms);
  if (st != JL_OK || n_keys == 0) return st;
  if (key_dtype == JL_BF16 && jlk::quantize_tc_supported(m, d, n_keys, key_stride, K)) {
    return from_cuda(jlk::launch_quantize_tc(
        reinterpret_cast<const uint16_t *>(K), n_keys, key_stride, S, m, d,
        signs, norms, (cudaStream_t)stream));
  }
  return from_cuda(jlk::launch_quantize_simt(K, key_dtype == JL_F32, n_keys,
                                             key_stride, S, m, d, signs, norms,
                                             (cudaStream_t)stream));
}

int jl_dequantize_keys(const uint32_t *signs, const uint16_t *norms, int64_t n_keys,
                       const uint16_t *S, int m, int d, uint16_t *out, jl_stream_t stream) {
  if (n_keys < 0) return JL_ERR_INVALID_ARG;
  if (!supported_md(m, d)) return JL_ERR_UNSUPPORTED;
  if (n_keys == 0) return JL_OK;
  if (!signs || !norms || !S || !out) return JL_ERR_INVALID_ARG;
  if (!aligned(signs, 16) || !aligned(norms, 2) || !aligned(S, 16) || !aligned(out, 16))
    return JL_ERR_INVALID_ARG;
  if (n_keys >= ((int64_t)1 << 40)) return JL_ERR_UNSUPPORTED;
  return from_cuda(jlk::launch_dequantize_tc(signs, norms, n_keys, S, m, d, out,
                                             (cudaStream_t)stream));
}

size_t jl_search_workspace_bytes(int n_queries, int m, int d, int k) {
  if (n_queries < 0 || k < 1 || k > JL_SEARCH_MAX_K || !supported_md(m, d)) return 0;
  return jlk::search_workspace_bytes(n_queries, m, k);
}

int jl_search_topk(const void *Q, jl_dtype q_dtype, int n_queries, const uint16_t *S, int m,
                   int d, const uint32_t *signs, const uint16_t *norms, int64_t n_index, int k,
                   int32_t *out_index, float *out_scores, void *workspace,
                   size_t workspace_bytes, jl_stream_t stream) {
  if (q_dtype != JL_BF16 && q_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (n_queries < 0 || n_index < 1 || k < 1 || k > JL_SEARCH_MAX_K) return JL_ERR_INVALID_ARG;
  if (!supported_md(m, d)) return JL_ERR_UNSUPPORTED;
  if (n_index >= ((int64_t)1 << 31)) return JL_ERR_UNSUPPORTED;
  if (n_queries == 0) return JL_OK;
  if (!Q || !S || !signs || !norms || !out_index || !out_scores) return JL_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(S, 16) || !aligned(signs, 16) || !aligned(norms, 2) ||
      !aligned(out_index, 4) || !aligned(out_scores, 4))
    return JL_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) ||
      workspace_bytes < jlk::search_workspace_bytes(n_queries, m, k))
    return JL_ERR_WORKSPACE;
  return from_cuda(jlk::launch_search(Q, q_dtype == JL_F32, n_queries, S, m, d, signs, norms,
                                      n_index, k, out_index, out_scores, workspace,
                                      (cudaStream_t)stream));
}

size_t jl_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int m,
                                 int d) {
  jlk::DecodePlan p;
  if (B == 0) return 0;
  if (!jlk::make_decode_plan(B, Hq, Hkv, T, m, d, &p)) return 0;
  return p.total_bytes;
}

int jl_decode_attention(const void *Q, jl_dtype q_dtype, const uint16_t *S,
                        const uint32_t *signs, const uint16_t *norms,
                        const uint16_t *V, int B, int Hq, int Hkv, int64_t T,
                        int m, int d, float softmax_scale, uint16_t *out,
                        float *scores, void *workspace, size_t workspace_bytes,
                        jl_stream_t stream) {
  jlk::DecodePlan p;
  bool empty = false;
  const int st = jlk::validate_decode(Q, q_dtype, S, signs, norms, V, B, Hq, Hkv, T, m, d,
                                      softmax_scale, out, scores, &p, &empty);
  if (st != JL_OK || empty) return st;
  if (!workspace || workspace_bytes < p.total_bytes || !aligned(workspace, 256))
    return JL_ERR_WORKSPACE;
  return from_cuda(jlk::launch_decode(p, Q, q_dtype == JL_F32, S, signs, norms,
                                      V, softmax_scale, out, scores, workspace,
                                      (cudaStream_t)stream));
}

int jl_decode_attention_state(const void *Q, jl_dtype q_dtype, const uint16_t *S,
                              const uint32_t *signs, const uint16_t *norms,
                              const uint16_t *V, int B, int Hq, int Hkv, int64_t T,
                              int m, int d, float softmax_scale, float *state,
                              float *scores, void *workspace, size_t workspace_bytes,
                              jl_stream_t stream) {
  jlk::DecodePlan p;
  bool empty = false;
  // the state buffer takes the output's checks (non-null, 4-byte aligned)
  const int st = jlk::validate_decode(Q, q_dtype, S, signs, norms, V, B, Hq, Hkv, T, m, d,
                                      softmax_scale, reinterpret_cast<const uint16_t *>(state),
                                      scores, &p, &empty);
  if (st != JL_OK || empty) return st;
  if (!workspace || workspace_bytes < p.total_bytes || !aligned(workspace, 256))
    return JL_ERR_WORKSPACE;
  return from_cuda(jlk::launch_decode(p, Q, q_dtype == JL_F32, S, signs, norms, V,
                                      softmax_scale, nullptr, scores, workspace,
                                      (cudaStream_t)stream, state));
}

int jl_merge_attention_states(const float *states, int R, int64_t rows, int d,
                              uint16_t *out, jl_stream_t stream) {
  if (R < 1 || R > 65536 || rows < 0 || rows >= ((int64_t)1 << 31)) return JL_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return JL_ERR_UNSUPPORTED;
  if (rows == 0) return JL_OK;
  if (!states || !out || !aligned(states, 4) || !aligned(out, 4)) return JL_ERR_INVALID_ARG;
  return from_cuda(jlk::launch_merge_states(states, R, rows, d, out, (cudaStream_t)stream));
}

size_t jl_decode_paged_workspace_bytes(int B, int Hq, int Hkv, int64_t max_len, int m,
                                       int d) {
  jlk::DecodePlan p;
  if (B == 0) return 0;
  if (!jlk::make_paged_plan(B, Hq, Hkv, max_len, m, d, &p)) return 0;
  return p.total_bytes;
}

int jl_decode_attention_paged(
    const void *Q, jl_dtype q_dtype, const void *K_new, jl_dtype k_dtype,
    const uint16_t *V_new, const uint16_t *S, uint32_t *sign_pages,
    uint16_t *norm_pages, uint16_t *value_pages, int num_pages, int page_tokens,
    const int32_t *block_table, int max_pages, const int32_t *seq_lens, int B, int Hq,
    int Hkv, int64_t max_len, int m, int d, float softmax_scale, uint16_t *out,
    float *scores, void *workspace, size_t workspace_bytes, jl_stream_t stream) {
  if (q_dtype != JL_BF16 && q_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (K_new && k_dtype != JL_BF16 && k_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || max_len < 1 || Hq % Hkv != 0) return JL_ERR_INVALID_ARG;
  if (num_pages < 1 || max_pages < 1 || page_tokens < 32 || page_tokens % 32 != 0)
    return JL_ERR_INVALID_ARG;
  if ((int64_t)max_pages * page_tokens < max_len) return JL_ERR_INVALID_ARG;
  if (!supported_md(m, d)) return JL_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale)) return JL_ERR_INVALID_ARG;
  if (B == 0) return JL_OK;
  if (!Q || !S || !sign_pages || !norm_pages || !value_pages || !block_table || !seq_lens ||
      !out)
    return JL_ERR_INVALID_ARG;
  if (K_new && !V_new) return JL_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(S, 16) || !aligned(sign_pages, 16) ||
      !aligned(norm_pages, 16) || !aligned(value_pages, 16) || !aligned(out, 4) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || (K_new && !aligned(K_new, 16)) ||
      (V_new && !aligned(V_new, 16)) || (scores && !aligned(scores, 4)))
    return JL_ERR_INVALID_ARG;
  jlk::DecodePlan p;
  if (!jlk::make_paged_plan(B, Hq, Hkv, max_len, m, d, &p)) return JL_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < p.total_bytes || !aligned(workspace, 256))
    return JL_ERR_WORKSPACE;
  jlk::PagedArgs a;
  a.Q = Q; a.q_f32 = q_dtype == JL_F32;
  a.K_new = K_new; a.k_f32 = k_dtype == JL_F32; a.V_new = V_new; a.S = S;
  a.sign_pages = sign_pages; a.norm_pages = norm_pages; a.value_pages = value_pages;
  a.num_pages = num_pages; a.page_tokens = page_tokens;
  a.block_table = block_table; a.max_pages = max_pages; a.seq_lens = seq_lens;
  a.softmax_scale = softmax_scale; a.out = out; a.scores = scores; a.workspace = workspace;
  return from_cuda(jlk::launch_decode_paged(p, a, (cudaStream_t)stream));
}

int jl_turbo_codebook(int d, int mse_bits, float *centroids) {
  if (!centroids) return JL_ERR_INVALID_ARG;
  if (d < 3 || d > 4096 || mse_bits < 1 || mse_bits > JL_TURBO_MAX_MSE_BITS)
    return JL_ERR_UNSUPPORTED;
  return jlk::turbo_codebook(d, mse_bits, centroids, nullptr) ? JL_OK : JL_ERR_UNSUPPORTED;
}

size_t jl_turbo_rotation_workspace_bytes(int d) { return jlk::turbo_rotation_workspace_bytes(d); }

int jl_turbo_rotation_init(uint16_t *Pi, float *Pinv, int d, uint64_t seed, void *workspace,
                           size_t workspace_bytes, jl_stream_t stream) {
  if (d != 64 && d != 128) return JL_ERR_UNSUPPORTED;
  if (!Pi || !Pinv || !aligned(Pi, 16) || !aligned(Pinv, 16)) return JL_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) ||
      workspace_bytes < jlk::turbo_rotation_workspace_bytes(d))
    return JL_ERR_WORKSPACE;
  return from_cuda(
      jlk::launch_turbo_rotation(Pi, Pinv, d, seed, workspace, (cudaStream_t)stream));
}

int jl_turbo_quantize_keys(const void *K, jl_dtype key_dtype, int64_t n_keys,
                           int64_t key_stride, const uint16_t *Pi, const uint16_t *S, int m,
                           int d, int mse_bits, uint32_t *codes, uint16_t *norms,
                           jl_stream_t stream) {
  if (key_dtype != JL_BF16 && key_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (n_keys < 0) return JL_ERR_INVALID_ARG;
  if (key_dtype != JL_BF16 || !turbo_md(m, d) || mse_bits < 1 ||
      mse_bits > JL_TURBO_MAX_MSE_BITS)
    return JL_ERR_UNSUPPORTED;
  if (n_keys == 0) return JL_OK;
  if (!K || !Pi || !S || !codes || !norms || key_stride < d) return JL_ERR_INVALID_ARG;
  if (!aligned(K, 16) || ((size_t)key_stride * 2) % 16 != 0 || !aligned(Pi, 16) ||
      !aligned(S, 16) || !aligned(codes, 16) || !aligned(norms, 4))
    return JL_ERR_INVALID_ARG;
  if (n_keys >= ((int64_t)1 << 31) || key_stride >= ((int64_t)1 << 39)) return JL_ERR_UNSUPPORTED;
  return from_cuda(jlk::launch_turbo_quantize(reinterpret_cast<const uint16_t *>(K), n_keys,
                                              key_stride, Pi, S, m, d, mse_bits, codes, norms,
                                              (cudaStream_t)stream));
}

size_t jl_turbo_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int m, int d,
                                       int mse_bits) {
  jlk::DecodePlan p;
  if (B == 0) return 0;
  if (!jlk::make_turbo_decode_plan(B, Hq, Hkv, T, m, d, mse_bits, &p)) return 0;
  return p.total_bytes;
}

int jl_turbo_decode_attention(const void *Q, jl_dtype q_dtype, const float *Pinv,
                              const uint16_t *S, const uint32_t *codes, const uint16_t *norms,
                              const uint16_t *V, int B, int Hq, int Hkv, int64_t T, int m,
                              int d, int mse_bits, float softmax_scale, uint16_t *out,
                              float *scores, void *workspace, size_t workspace_bytes,
                              jl_stream_t stream) {
  if (q_dtype != JL_BF16 && q_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv != 0) return JL_ERR_INVALID_ARG;
  if (!turbo_md(m, d) || mse_bits < 1 || mse_bits > JL_TURBO_MAX_MSE_BITS)
    return JL_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale)) return JL_ERR_INVALID_ARG;
  if (B == 0) return JL_OK;
  if (!Q || !Pinv || !S || !codes || !norms || !V || !out) return JL_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(Pinv, 16) || !aligned(S, 16) || !aligned(codes, 16) ||
      !aligned(norms, 16) || !aligned(V, 16) || !aligned(out, 4) ||
      (scores && !aligned(scores, 4)))
    return JL_ERR_INVALID_ARG;
  jlk::DecodePlan p;
  if (!jlk::make_turbo_decode_plan(B, Hq, Hkv, T, m, d, mse_bits, &p)) return JL_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < p.total_bytes || !aligned(workspace, 256))
    return JL_ERR_WORKSPACE;
  double walsh[4];
  if (!jlk::turbo_codebook(d, mse_bits, nullptr, walsh)) return JL_ERR_UNSUPPORTED;
  return from_cuda(jlk::launch_turbo_decode(p, mse_bits, Q, q_dtype == JL_F32, Pinv, S, codes,
                                            norms, V, walsh, softmax_scale, out, scores,
                                            workspace, (cudaStream_t)stream));
}

size_t jl_turbo_decode_paged_workspace_bytes(int B, int Hq, int Hkv, int64_t max_len, int m,
                                             int d, int mse_bits) {
  return jl_turbo_decode_workspace_bytes(B, Hq, Hkv, max_len, m, d, mse_bits);
}

int jl_turbo_decode_attention_paged(
    const void *Q, jl_dtype q_dtype, const void *K_new, jl_dtype k_dtype, const uint16_t *V_new,
    const uint16_t *Pi, const float *Pinv, const uint16_t *S, uint32_t *code_pages,
    uint16_t *norm_pages, uint16_t *value_pages, int num_pages, int page_tokens,
    const int32_t *block_table, int max_pages, const int32_t *seq_lens, int B, int Hq, int Hkv,
    int64_t max_len, int m, int d, int mse_bits, float softmax_scale, uint16_t *out,
    float *scores, void *workspace, size_t workspace_bytes, jl_stream_t stream) {
  if (q_dtype != JL_BF16 && q_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (K_new && k_dtype != JL_BF16 && k_dtype != JL_F32) return JL_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || max_len < 1 || Hq % Hkv != 0) return JL_ERR_INVALID_ARG;
  if (num_pages < 1 || max_pages < 1 || page_tokens < 32 || page_tokens % 32 != 0)
    return JL_ERR_INVALID_ARG;
  if ((int64_t)max_pages * page_tokens < max_len) return JL_ERR_INVALID_ARG;
  if (!turbo_md(m, d) || mse_bits < 1 || mse_bits > JL_TURBO_MAX_MSE_BITS)
    return JL_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale)) return JL_ERR_INVALID_ARG;
  if (B == 0) return JL_OK;
  if (!Q || !Pinv || !S || !code_pages || !norm_pages || !value_pages || !block_table ||
      !seq_lens || !out)
    return JL_ERR_INVALID_ARG;
  if (K_new && (!V_new || !Pi)) return JL_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(Pinv, 16) || !aligned(S, 16) || !aligned(code_pages, 16) ||
      !aligned(norm_pages, 16) || !aligned(value_pages, 16) || !aligned(out, 4) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || (K_new && !aligned(K_new, 16)) ||
      (V_new && !aligned(V_new, 16)) || (Pi && !aligned(Pi, 16)) ||
      (scores && !aligned(scores, 4)))
    return JL_ERR_INVALID_ARG;
  jlk::DecodePlan p;
  if (!jlk::make_turbo_decode_plan(B, Hq, Hkv, max_len, m, d, mse_bits, &p))
    return JL_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < p.total_bytes || !aligned(workspace, 256))
    return JL_ERR_WORKSPACE;
  jlk::TurboPagedArgs t;
  t.Pi = Pi;
  t.Pinv = Pinv;
  if (!jlk::turbo_codebook(d, mse_bits, nullptr, t.walsh) ||
      !jlk::turbo_magnitudes(d, mse_bits, t.mag, t.pos_thr))
    return JL_ERR_UNSUPPORTED;
  jlk::PagedArgs a;
  a.Q = Q; a.q_f32 = q_dtype == JL_F32;
  a.K_new = K_new; a.k_f32 = k_dtype == JL_F32; a.V_new = V_new; a.S = S;
  a.sign_pages = code_pages; a.norm_pages = norm_pages; a.value_pages = value_pages;
  a.num_pages = num_pages; a.page_tokens = page_tokens;
  a.block_table = block_table; a.max_pages = max_pages; a.seq_lens = seq_lens;
  a.softmax_scale = softmax_scale; a.out = out; a.scores = scores; a.workspace = workspace;
  return from_cuda(jlk::launch_turbo_decode_paged(p, mse_bits, a, t, (cudaStream_t)stream));
}

int jl_turbo_dequant_basis(const float *Pinv, const uint16_t *S, int m, int d,
                           uint16_t *basis, jl_stream_t stream) {
  if (!turbo_md(m, d)) return JL_ERR_UNSUPPORTED;
  if (!Pinv || !S || !basis) return JL_ERR_INVALID_ARG;
  if (!aligned(Pinv, 16) || !aligned(S, 16) || !aligned(basis, 16)) return JL_ERR_INVALID_ARG;
  return from_cuda(jlk::launch_turbo_dequant_basis(Pinv, S, m, d, basis, (cudaStream_t)stream));
}

int jl_turbo_dequantize_keys(const uint32_t *codes, const uint16_t *norms, int64_t n_keys,
                             const uint16_t *basis, int m, int d, int mse_bits, uint16_t *out,
                             jl_stream_t stream) {
  if (n_keys < 0) return JL_ERR_INVALID_ARG;
  if (!turbo_md(m, d) || mse_bits < 1 || mse_bits > JL_TURBO_MAX_MSE_BITS)
    return JL_ERR_UNSUPPORTED;
  if (n_keys == 0) return JL_OK;
  if (!codes || !norms || !basis || !out) return JL_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(norms, 4) || !aligned(basis, 16) || !aligned(out, 16))
    return JL_ERR_INVALID_ARG;
  if (n_keys >= ((int64_t)1 << 40)) return JL_ERR_UNSUPPORTED;
  return from_cuda(jlk::launch_turbo_dequantize(codes, norms, n_keys, basis, m, d, mse_bits, out,
                                                (cudaStream_t)stream));
}

int jl_test_drop_copies(int enable, uint64_t wait_limit_ns) {
  if (enable != 0 && enable != 1) return JL_ERR_INVALID_ARG;
  unsigned long long lim = wait_limit_ns ? (unsigned long long)wait_limit_ns : jlk::WAIT_LIMIT_NS;
  if (lim < 1000ull || lim > jlk::WAIT_LIMIT_NS) return JL_ERR_INVALID_ARG;
  jlk::g_wait_limit_ns.store(lim, std::memory_order_relaxed);
  jlk::g_drop_copies.store(enable, std::memory_order_relaxed);
  return JL_OK;
}

int jl_build_flags(void) {
#ifdef JL_DEBUG_INDEX
  return JL_BUILD_INDEX_CHECKS;
#else
  return 0;
#endif
}

int jl_device_error(int *code, jl_stream_t stream) {
  if (!code) return JL_ERR_INVALID_ARG;
  *code = 0;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
    return JL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, jlk::g_device_error, sizeof(int)) != cudaSuccess)
    return JL_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(jlk::g_device_error, &zero, sizeof(int)) !=
        cudaSuccess)
      return JL_ERR_CUDA;
  }
  *code = v;
  return v ? JL_ERR_DEVICE : JL_OK;
}

}  // extern "C"
