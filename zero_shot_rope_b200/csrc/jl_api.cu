// Host side of the C ABI declared in include/jetlong.h: argument validation,
// status reporting and kernel dispatch.  Nothing here computes attention.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/jetlong.h"
#include "jl_common.cuh"

namespace jl {
cudaError_t launch_simt_prefill(bool bf16, int D, const void *q, const void *k, const void *v, void *out,
                                float *lse, const int32_t *cu, const int32_t *cu_k, int batch, int T_total,
                                int Tk, int Hq, int Hkv, long long w_pre, int w0, int window,
                                const InvFreq &inv, int plain, cudaStream_t st);
struct DecodePlan {
  int nsplit;
  int chunk;
  size_t smem_bytes;
};
DecodePlan decode_plan(int batch, int Hq, int Hkv, int D, int max_seqlen, int elem);
size_t decode_partial_rows(int batch, int Hq, int Hkv, int D, int max_seqlen);
size_t decode_plan_tab_bytes();
cudaError_t launch_decode(bool bf16, int D, int GS, const void *q, const void *kc, const void *vc,
                          const int32_t *seqlens, int B, int Lcap, int max_seqlen, int Hq, int Hkv,
                          long long w_pre, int w0, int window, const InvFreq &inv, int plain, float *part_o,
                          float *part_ml, int2 *plan_tab, int *err, void *out, float *lse, cudaStream_t st);
size_t tc_prefill_workspace(int batch, int T_total, int Hq, int Hkv, int D, uint32_t flags);
cudaError_t launch_tc_prefill(const void *q, const void *k, const void *v, void *out, float *lse,
                              const int32_t *cu, const int32_t *cu_k, int batch, int T_total, int Tk,
                              int max_seqlen, int Hq, int Hkv, int D, long long w_pre, int w0, int window,
                              const InvFreq &inv, int plain, uint32_t flags, void *ws, size_t ws_bytes,
                              cudaStream_t st, const char **why);
}  // namespace jl

namespace {

thread_local char g_err[320] = "";

jl_status fail(jl_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

jl_status ok() {
  g_err[0] = '\0';
  return JL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

jl::InvFreq make_inv_freq(int D, double theta) {
  jl::InvFreq f;
  for (int k = 0; k < JL_MAX_HALF; ++k) f.v[k] = 0.0;
  for (int k = 0; k < D / 2; ++k) f.v[k] = std::pow(theta, -2.0 * (double)k / (double)D);
  return f;
}

jl_status check_heads(int32_t Hq, int32_t Hkv, int32_t D) {
  if (Hq <= 0 || Hkv <= 0) return fail(JL_ERR_INVALID_ARG, "head counts must be positive (Hq=%d, Hkv=%d)", Hq, Hkv);
  if (Hq % Hkv != 0) return fail(JL_ERR_INVALID_ARG, "n_q_heads (%d) is not a multiple of n_kv_heads (%d)", Hq, Hkv);
  if (D != 64 && D != 128) return fail(JL_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", D);
  return JL_OK;
}

// The kernels put one head (prefill: a query head or a pair of them; decode:
// a kv head) per y-block of their grid, whose extent is at most 65535.
constexpr int32_t kMaxGridY = 65535;

jl_status check_method(int64_t w_pre, int32_t w0, double theta) {
  if (w_pre < 1) return fail(JL_ERR_INVALID_ARG, "w_pretrained must be >= 1 (got %lld)", (long long)w_pre);
  if (w0 < 0) return fail(JL_ERR_INVALID_ARG, "w0 must be >= 0 (got %d)", w0);
  if (!(theta > 0.0) || !std::isfinite(theta)) return fail(JL_ERR_INVALID_ARG, "rope_theta must be finite and > 0");
  return JL_OK;
}

jl_status cuda_fail(cudaError_t e, const char *what) {
  return fail(JL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace jl {
// Record a message for jl_last_error() from other translation units.
void set_last_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}
}  // namespace jl

extern "C" {

const char *jl_status_string(jl_status s) {
  switch (s) {
    case JL_OK: return "JL_OK";
    case JL_ERR_INVALID_ARG: return "JL_ERR_INVALID_ARG";
    case JL_ERR_UNSUPPORTED: return "JL_ERR_UNSUPPORTED";
    case JL_ERR_CUDA: return "JL_ERR_CUDA";
    case JL_ERR_WORKSPACE: return "JL_ERR_WORKSPACE";
  }
  return "JL_STATUS_UNKNOWN";
}

const char *jl_last_error(void) { return g_err; }

const char *jl_version(void) { return "jetlong-b200 0.1 sm_100a"; }

jl_status jl_group_size(int64_t L, int64_t w_pretrained, int64_t *G_out) {
  if (G_out == nullptr) return fail(JL_ERR_INVALID_ARG, "G_out is NULL");
  if (L < 0) return fail(JL_ERR_INVALID_ARG, "L must be >= 0 (got %lld)", (long long)L);
  if (w_pretrained < 1) return fail(JL_ERR_INVALID_ARG, "w_pretrained must be >= 1 (got %lld)", (long long)w_pretrained);
  // ceil without overflow for L near INT64_MAX
  const int64_t g = L / w_pretrained + (L % w_pretrained != 0 ? 1 : 0);
  *G_out = g < 1 ? 1 : g;
  return ok();
}

size_t jl_bifocal_prefill_workspace_size(int32_t batch, int32_t total_tokens, int32_t n_q_heads,
                                         int32_t n_kv_heads, int32_t head_dim, jl_dtype dtype,
                                         uint32_t flags) {
  if (batch < 0 || total_tokens < 0 || n_q_heads <= 0 || n_kv_heads <= 0) return 0;
  if (n_q_heads % n_kv_heads != 0) return 0;
  const bool tc_shape = head_dim == 128 || head_dim == 64;
  if (dtype != JL_BF16 || (flags & JL_FLAG_SIMT) || !tc_shape) return 0;
  return jl::tc_prefill_workspace(batch, total_tokens, n_q_heads, n_kv_heads, head_dim, flags);
}

jl_status jl_bifocal_prefill_kv(const void *q, const void *k, const void *v, void *out, float *lse,
                                const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t batch,
                                int32_t total_q, int32_t total_k, int32_t max_seqlen_q, int32_t n_q_heads,
                                int32_t n_kv_heads, int32_t head_dim, int64_t w_pretrained, int32_t w0,
                                int32_t window, double rope_theta, jl_dtype dtype, uint32_t flags,
                                void *workspace, size_t workspace_bytes, void *stream) {
  jl_status s;
  if ((s = check_heads(n_q_heads, n_kv_heads, head_dim)) != JL_OK) return s;
  if (n_q_heads > kMaxGridY)
    return fail(JL_ERR_UNSUPPORTED, "n_q_heads %d exceeds %d per call", n_q_heads, kMaxGridY);
  if ((s = check_method(w_pretrained, w0, rope_theta)) != JL_OK) return s;
  if (window < 0) return fail(JL_ERR_INVALID_ARG, "window must be >= 0 (0: no window), got %d", window);
  if (dtype != JL_BF16 && dtype != JL_FP32) return fail(JL_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (flags & ~(uint32_t)(JL_FLAG_PLAIN_CAUSAL | JL_FLAG_SIMT | JL_FLAG_PREROTATE_K))
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (batch < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0)
    return fail(JL_ERR_INVALID_ARG, "batch, token counts and max_seqlen must be >= 0");
  if (batch == 0 || total_q == 0) return ok();  // nothing to attend
  if (batch > 65535)  // the kernels' grid takes one z-block per sequence
    return fail(JL_ERR_UNSUPPORTED, "batch %d exceeds 65535 sequences per call", batch);
  if (total_k < total_q)
    return fail(JL_ERR_INVALID_ARG, "total_k (%d) < total_q (%d): every sequence needs Lq <= Lk", total_k, total_q);
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return fail(JL_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr)
    return fail(JL_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned16(lse)))
    return fail(JL_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (max_seqlen_q == 0 || max_seqlen_q > total_q)
    return fail(JL_ERR_INVALID_ARG, "max_seqlen must be in [1, total query tokens] (got %d)", max_seqlen_q);

  const jl::InvFreq inv = make_inv_freq(head_dim, rope_theta);
  const int plain = (flags & JL_FLAG_PLAIN_CAUSAL) ? 1 : 0;
  cudaStream_t st = (cudaStream_t)stream;
  // tensor cores for bf16 at head_dim 64 and 128; the SIMT kernel otherwise
  const bool tc_shape = head_dim == 128 || head_dim == 64;
  const bool use_simt = dtype == JL_FP32 || (flags & JL_FLAG_SIMT) || !tc_shape;
  if (use_simt) {
    cudaError_t e = jl::launch_simt_prefill(dtype == JL_BF16, head_dim, q, k, v, out, lse, cu_seqlens_q,
                                            cu_seqlens_k, batch, total_q, total_k, n_q_heads, n_kv_heads,
                                            w_pretrained, w0, window, inv, plain, st);
    return e == cudaSuccess ? ok() : cuda_fail(e, "SIMT prefill launch");
  }
  const size_t need = jl::tc_prefill_workspace(batch, total_k, n_q_heads, n_kv_heads, head_dim, flags);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(JL_ERR_WORKSPACE, "prefill needs %zu workspace bytes (got %zu)", need, workspace_bytes);
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(JL_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const char *why = nullptr;
  cudaError_t e = jl::launch_tc_prefill(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                        max_seqlen_q, n_q_heads, n_kv_heads, head_dim, w_pretrained, w0, window,
                                        inv, plain, flags, workspace, workspace_bytes, st, &why);
  return e == cudaSuccess ? ok() : cuda_fail(e, why ? why : "tensor-core prefill launch");
}

jl_status jl_bifocal_prefill(const void *q, const void *k, const void *v, void *out, float *lse,
                             const int32_t *cu_seqlens, int32_t batch, int32_t total_tokens,
                             int32_t max_seqlen, int32_t n_q_heads, int32_t n_kv_heads,
                             int32_t head_dim, int64_t w_pretrained, int32_t w0, double rope_theta,
                             jl_dtype dtype, uint32_t flags, void *workspace,
                             size_t workspace_bytes, void *stream) {
  // every token of every sequence is a query: the key prefix sums are the
  // query prefix sums
  return jl_bifocal_prefill_kv(q, k, v, out, lse, cu_seqlens, cu_seqlens, batch, total_tokens, total_tokens,
                               max_seqlen, n_q_heads, n_kv_heads, head_dim, w_pretrained, w0, 0, rope_theta,
                               dtype, flags, workspace, workspace_bytes, stream);
}

size_t jl_bifocal_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                        int32_t head_dim, int32_t max_seqlen) {
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || max_seqlen < 0) return 0;
  if (n_q_heads % n_kv_heads != 0) return 0;
  // one layout serves every dtype and both decode kernels
  const size_t rows = jl::decode_partial_rows(batch, n_q_heads, n_kv_heads, head_dim, max_seqlen);
  return 256 + align256(rows * head_dim * sizeof(float)) + align256(rows * 2 * sizeof(float)) +
         align256(jl::decode_plan_tab_bytes());
}

jl_status jl_bifocal_decode_window(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *seqlens, int32_t batch, int32_t cache_capacity,
                                   int32_t max_seqlen, int32_t n_q_heads, int32_t n_kv_heads,
                                   int32_t head_dim, int64_t w_pretrained, int32_t w0, int32_t window,
                                   double rope_theta, void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, jl_dtype dtype, uint32_t flags, void *stream) {
  jl_status s;
  if (window < 0) return fail(JL_ERR_INVALID_ARG, "window must be >= 0 (0: no window), got %d", window);
  if ((s = check_heads(n_q_heads, n_kv_heads, head_dim)) != JL_OK) return s;
  if (n_kv_heads > kMaxGridY)
    return fail(JL_ERR_UNSUPPORTED, "n_kv_heads %d exceeds %d per call", n_kv_heads, kMaxGridY);
  const int gs = n_q_heads / n_kv_heads;
  if (gs != 1 && gs != 2 && gs != 4 && gs != 8)
    return fail(JL_ERR_UNSUPPORTED, "decode supports n_q_heads / n_kv_heads in {1,2,4,8} (got %d)", gs);
  if ((s = check_method(w_pretrained, w0, rope_theta)) != JL_OK) return s;
  if (dtype != JL_BF16 && dtype != JL_FP32) return fail(JL_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (flags & ~(uint32_t)JL_FLAG_PLAIN_CAUSAL) return fail(JL_ERR_INVALID_ARG, "unknown or prefill-only flag bits 0x%x", flags);
  if (batch < 0) return fail(JL_ERR_INVALID_ARG, "batch must be >= 0");
  if (batch == 0) return ok();
  if (batch > 65535)  // the kernels' grid takes one z-block per sequence
    return fail(JL_ERR_UNSUPPORTED, "batch %d exceeds 65535 sequences per call", batch);
  if (cache_capacity < 1 || max_seqlen < 1 || max_seqlen > cache_capacity)
    return fail(JL_ERR_INVALID_ARG, "need 1 <= max_seqlen <= cache_capacity (got %d, %d)", max_seqlen, cache_capacity);
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || out == nullptr || seqlens == nullptr)
    return fail(JL_ERR_INVALID_ARG, "q, k_cache, v_cache, seqlens and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return fail(JL_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t need = jl_bifocal_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_seqlen);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(JL_ERR_WORKSPACE, "decode needs %zu workspace bytes (got %zu)", need, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(JL_ERR_WORKSPACE, "workspace must be 256-byte aligned");

  const size_t rows = jl::decode_partial_rows(batch, n_q_heads, n_kv_heads, head_dim, max_seqlen);
  int *err = (int *)workspace;
  float *part_o = (float *)((char *)workspace + 256);
  float *part_ml = (float *)((char *)workspace + 256 + align256(rows * head_dim * sizeof(float)));
  int2 *plan_tab = (int2 *)((char *)part_ml + align256(rows * 2 * sizeof(float)));
  const jl::InvFreq inv = make_inv_freq(head_dim, rope_theta);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e == cudaSuccess)
    e = jl::launch_decode(dtype == JL_BF16, head_dim, gs, q, k_cache, v_cache, seqlens, batch, cache_capacity,
                          max_seqlen, n_q_heads, n_kv_heads, w_pretrained, w0, window, inv,
                          (flags & JL_FLAG_PLAIN_CAUSAL) ? 1 : 0, part_o, part_ml, plan_tab, err, out, lse, st);
  return e == cudaSuccess ? ok() : cuda_fail(e, "decode launch");
}

jl_status jl_bifocal_decode(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, int32_t batch, int32_t cache_capacity,
                            int32_t max_seqlen, int32_t n_q_heads, int32_t n_kv_heads,
                            int32_t head_dim, int64_t w_pretrained, int32_t w0, double rope_theta,
                            void *out, float *lse, void *workspace, size_t workspace_bytes,
                            jl_dtype dtype, uint32_t flags, void *stream) {
  return jl_bifocal_decode_window(q, k_cache, v_cache, seqlens, batch, cache_capacity, max_seqlen, n_q_heads,
                                  n_kv_heads, head_dim, w_pretrained, w0, 0, rope_theta, out, lse, workspace,
                                  workspace_bytes, dtype, flags, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- test hooks
namespace jl {
cudaError_t set_wait_limit_prefill(unsigned long long ns);
cudaError_t set_wait_limit_decode_tc(unsigned long long ns);
cudaError_t set_wait_limit_decode(unsigned long long ns);
}  // namespace jl

extern "C" int jl_debug_set_wait_limit(unsigned long long ns) {
  if (ns == 0) ns = 2000000000ull;
  cudaError_t e = jl::set_wait_limit_prefill(ns);
  if (e == cudaSuccess) e = jl::set_wait_limit_decode_tc(ns);
  if (e == cudaSuccess) e = jl::set_wait_limit_decode(ns);
  if (e != cudaSuccess) {
    fail(JL_ERR_CUDA, "setting the wait limit failed: %s", cudaGetErrorString(e));
    return -1;
  }
  return 0;
}

extern "C" void jl_debug_angle_cs(int32_t n, double inv_freq, float *c, float *s) {
  jl::angle_cs(n, inv_freq, *c, *s);
}
