/*
 * jetlong.h — C ABI of the Dynamic Bifocal RoPE attention library (sm_100a).
 *
 * The method: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
 * RoPE" (Tang, Wang, Gu, Han, Cai).  Citations below name sections of its
 * technical summary on gist.science ("Resumo Técnico: Jet-Long", Portuguese;
 * the French "Résumé Technique : Jet-Long" repeats it):
 *   §1 "RoPE Bifocal Dinâmico"   — local window w0, remote map f, group size G;
 *   §2 "Mecanismos de Eficiência de Inferência" — the on-the-fly correction
 *       rotation and the inclusion–exclusion attention merge.
 *
 * What every attention entry point computes (for each sequence of length L,
 * G = max(1, ceil(L / w_pretrained)), f(x) = floor(x / G), each query head h
 * reading kv head h / (Hq / Hkv), positions 0 .. L-1, d = p_i - p_j):
 *
 *   d < 0          : masked (causal)
 *   0 <= d < w0    : s_ij = <Q~_i, K~_j> / sqrt(D)                  (local window, base RoPE)
 *   d >= w0        : s_ij = <R(f(p_i)-p_i) Q~_i, R(f(p_j)-p_j) K~_j> / sqrt(D)   (remote, grouped)
 *   O_i = sum_j softmax_j(s_ij) V_j,   LSE_i = log sum_j exp(s_ij)
 *
 * Q~ and K~ arrive rotated by standard half-split RoPE at their absolute
 * position (pair k = (x_k, x_{k+D/2}), angle p * theta^(-2k/D)); V is not
 * rotated.  R(m) is that rotation by m positions.  This single masked softmax
 * is the exact value of the pages' three-pass inclusion–exclusion merge
 * (local/base + causal/grouped - local/grouped, LSE-weighted); the kernels
 * take the selection per score before the exponential instead of running
 * three passes.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them.  Integer arrays are int32 on the device.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronise.
 *  - Arguments are validated on the host before any launch; a rejected call
 *    returns JL_ERR_INVALID_ARG / JL_ERR_UNSUPPORTED / JL_ERR_WORKSPACE and has
 *    no side effect.  A failed launch returns JL_ERR_CUDA.  jl_last_error()
 *    gives a one-line reason for the most recent failure on the calling thread.
 *  - No C++ exception crosses this boundary; no call falls back to the CPU.
 */
#ifndef JETLONG_H
#define JETLONG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JL_OK = 0,
  JL_ERR_INVALID_ARG = 1, /* null pointer, bad size or inconsistent shapes   */
  JL_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim 96)    */
  JL_ERR_CUDA = 3,        /* a CUDA launch or driver call failed             */
  JL_ERR_WORKSPACE = 4    /* workspace missing, too small or misaligned      */
} jl_status;

typedef enum {
  JL_BF16 = 0, /* q, k, v, out in bfloat16; fp32 accumulation            */
  JL_FP32 = 1  /* q, k, v, out in float32; SIMT kernel, fp32 throughout   */
} jl_dtype;

/* flags (bitwise OR) */
#define JL_FLAG_PLAIN_CAUSAL 0x1u /* bifocal off: plain causal RoPE attention,
                                     the comparison mode (G forced to 1)      */
#define JL_FLAG_SIMT 0x2u         /* prefill: run the SIMT reference kernel
                                     instead of the tensor-core kernel       */
#define JL_FLAG_PREROTATE_K 0x4u  /* prefill, ablation of the in-tile key
                                     correction: a pre-pass writes the
                                     grouped keys R(f(j)-j) K~ of every key
                                     into the workspace (size it with this
                                     flag) and the grouped visits load them;
                                     same result, more HBM traffic           */

/* Human-readable name of a status code (static string). */
const char *jl_status_string(jl_status s);

/* One-line reason for the last non-JL_OK status returned on this thread
 * (static thread-local buffer; "" if none). */
const char *jl_last_error(void);

/* Library version string, e.g. "jetlong-b200 0.1 sm_100a". */
const char *jl_version(void);

/*
 * jl_group_size — dynamic group size, §1 "RoPE Bifocal Dinâmico", bullet
 * "Agrupamento Dinâmico":  G = max(1, ceil(L / w_pretrained)).
 *   L >= 0, w_pretrained >= 1, G_out non-NULL (host pointer), else
 *   JL_ERR_INVALID_ARG.  Exact integer arithmetic; L = 0 gives G = 1.
 *   Host-only; no CUDA call.
 */
jl_status jl_group_size(int64_t L, int64_t w_pretrained, int64_t *G_out);

/*
 * jl_bifocal_prefill_workspace_size — bytes of device workspace that
 * jl_bifocal_prefill needs for these sizes and flags (0 if none); for
 * jl_bifocal_prefill_kv pass the key token count as total_tokens.  The
 * workspace must be 256-byte aligned; its contents need no initialisation and
 * are scratch between calls.
 */
size_t jl_bifocal_prefill_workspace_size(int32_t batch, int32_t total_tokens,
                                         int32_t n_q_heads, int32_t n_kv_heads,
                                         int32_t head_dim, jl_dtype dtype,
                                         uint32_t flags);

/*
 * jl_bifocal_prefill — causal GQA prefill of a packed batch of sequences with
 * Dynamic Bifocal RoPE (§1) using the on-the-fly correction rotation and the
 * exact inclusion–exclusion merge (§2).
 *
 *   q           [T, Hq, D]   standard-RoPE queries, row-major, contiguous
 *   k           [T, Hkv, D]  standard-RoPE keys (the KV cache form)
 *   v           [T, Hkv, D]  values
 *   out         [T, Hq, D]   written for every token of every sequence
 *   lse         [Hq, T] fp32 natural-log LSE of the scaled scores, or NULL
 *   cu_seqlens  [batch + 1]  device int32 prefix sums, cu[0] = 0,
 *                            cu[batch] = total_tokens, non-decreasing; a
 *                            zero-length sequence is legal and writes nothing
 *   batch       <= 65535 sequences per call (JL_ERR_UNSUPPORTED beyond)
 *   max_seqlen  >= every sequence length (sizes the grid)
 *   head_dim    64 or 128;   n_q_heads % n_kv_heads == 0
 *   w_pretrained >= 1; w0 >= 0 (w0 = 0: every pair grouped; w0 >= L: none)
 *   rope_theta  > 0, the model's RoPE base
 *   dtype       JL_BF16 (tensor-core kernel, or SIMT with JL_FLAG_SIMT) or
 *               JL_FP32 (SIMT kernel)
 *   workspace   device buffer of at least
 *               jl_bifocal_prefill_workspace_size(...) bytes (may be NULL when
 *               that size is 0)
 * Positions are the in-sequence indices 0 .. L-1 of each packed sequence.
 * Pointers must be 16-byte aligned.
 */
jl_status jl_bifocal_prefill(const void *q, const void *k, const void *v,
                             void *out, float *lse,
                             const int32_t *cu_seqlens, int32_t batch,
                             int32_t total_tokens, int32_t max_seqlen,
                             int32_t n_q_heads, int32_t n_kv_heads,
                             int32_t head_dim, int64_t w_pretrained,
                             int32_t w0, double rope_theta, jl_dtype dtype,
                             uint32_t flags, void *workspace,
                             size_t workspace_bytes, void *stream);

/*
 * jl_bifocal_prefill_kv — prefill of new tokens against keys that include an
 * existing cache (chunked prefill; §2 "Rotação de Correção On-the-Fly":
 * generation streams across length boundaries and the cache of standard-RoPE
 * keys is never rewritten).
 *
 * Sequence s has Lk = cu_seqlens_k[s+1] - cu_seqlens_k[s] keys and values
 * (positions 0 .. Lk-1, rows cu_seqlens_k[s] .. of k and v) and
 * Lq = cu_seqlens_q[s+1] - cu_seqlens_q[s] <= Lk queries, which are the
 * newest tokens: positions Lk-Lq .. Lk-1.  G = G(Lk), the current length.
 *   q, out      [total_q, Hq, D];  lse [Hq, total_q] fp32 or NULL
 *   k, v        [total_k, Hkv, D]
 *   cu_seqlens_q, cu_seqlens_k   device int32 [batch + 1], each starting at 0
 *   max_seqlen_q >= every Lq
 *   window      0 for a global attention layer; W >= 1 for a sliding-window
 *               layer of a hybrid model ("Principais Contribuições" 4: the
 *               method carries over to hybrid attention stacks unchanged):
 *               keys at distance p_i - p_j >= W are hidden, the visible ones
 *               follow the bifocal rule with G = G(Lk).  W <= w0 is plain
 *               sliding-window RoPE attention.  Negative: JL_ERR_INVALID_ARG.
 *   workspace   >= jl_bifocal_prefill_workspace_size(batch, total_k, ...)
 * Other arguments as for jl_bifocal_prefill (which is this call with
 * cu_seqlens_k = cu_seqlens_q and window = 0).  Lq = 1 is one decode step.
 * The prefix sums live on the device and are not checked on the host: a
 * sequence with
 * Lq > Lk, or whose rows run past total_q / total_k, is skipped by the kernels
 * and its rows of out and lse are left unwritten.
 */
jl_status jl_bifocal_prefill_kv(const void *q, const void *k, const void *v,
                                void *out, float *lse,
                                const int32_t *cu_seqlens_q,
                                const int32_t *cu_seqlens_k, int32_t batch,
                                int32_t total_q, int32_t total_k,
                                int32_t max_seqlen_q, int32_t n_q_heads,
                                int32_t n_kv_heads, int32_t head_dim,
                                int64_t w_pretrained, int32_t w0,
                                int32_t window, double rope_theta,
                                jl_dtype dtype, uint32_t flags,
                                void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * jl_bifocal_decode_workspace_size — bytes of device workspace for
 * jl_bifocal_decode (split-KV partial results), 256-byte aligned, no
 * initialisation needed.
 */
size_t jl_bifocal_decode_workspace_size(int32_t batch, int32_t n_q_heads,
                                        int32_t n_kv_heads, int32_t head_dim,
                                        int32_t max_seqlen);

/*
 * jl_bifocal_decode — one generation step against a standard-RoPE KV cache
 * that is never rewritten (§2 "Rotação de Correção On-the-Fly": the
 * correction rotation is applied to the active query and the stored keys on
 * the fly; G is recomputed from the current length at every step).
 *
 *   q          [B, Hq, D]          query of the new token, standard RoPE at
 *                                  position L_b - 1
 *   k_cache    [B, Lcap, Hkv, D]   keys 0 .. L_b-1 (the new token's included)
 *   v_cache    [B, Lcap, Hkv, D]   values
 *   seqlens    [B] device int32    L_b, 1 <= L_b <= min(cache_capacity,
 *                                  max_seqlen); L_b = 0, or a value outside
 *                                  that range, writes zeros and LSE = -inf
 *   out        [B, Hq, D]          attention output (dtype of q)
 *   lse        [B, Hq] fp32 or NULL
 *   workspace  >= jl_bifocal_decode_workspace_size(...) bytes
 * head_dim 64 or 128; n_q_heads / n_kv_heads in {1, 2, 4, 8}; batch <= 65535.
 */
jl_status jl_bifocal_decode(const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *seqlens,
                            int32_t batch, int32_t cache_capacity,
                            int32_t max_seqlen, int32_t n_q_heads,
                            int32_t n_kv_heads, int32_t head_dim,
                            int64_t w_pretrained, int32_t w0,
                            double rope_theta, void *out, float *lse,
                            void *workspace, size_t workspace_bytes,
                            jl_dtype dtype, uint32_t flags, void *stream);

/*
 * jl_bifocal_decode_window — jl_bifocal_decode for a sliding-window layer of
 * a hybrid model ("Principais Contribuições" 4: the method carries over to
 * hybrid attention stacks unchanged).  The new query of sequence b attends to
 * the keys max(0, L_b - window) .. L_b - 1 only, scored by the bifocal rule
 * with G = G(L_b); window = 0 is jl_bifocal_decode.  The splits cover
 * min(max_seqlen, window) keys, so a narrow window costs what its keys cost.
 * All other arguments, the workspace size and the error behaviour are those
 * of jl_bifocal_decode; a negative window is JL_ERR_INVALID_ARG.
 */
jl_status jl_bifocal_decode_window(const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *seqlens,
                                   int32_t batch, int32_t cache_capacity,
                                   int32_t max_seqlen, int32_t n_q_heads,
                                   int32_t n_kv_heads, int32_t head_dim,
                                   int64_t w_pretrained, int32_t w0,
                                   int32_t window, double rope_theta,
                                   void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, jl_dtype dtype,
                                   uint32_t flags, void *stream);

/*
 * jl_bifocal_decode_noalloc — jl_bifocal_decode without a caller workspace.
 * (An addition of this library for callers that cannot allocate; the paper
 * has no counterpart.)
 *
 * Some callers cannot call cudaMalloc: a plugin hosted by a runtime that owns
 * the whole device-memory budget, or a latency-critical generation loop that
 * must not risk the implicit device synchronisation an allocation can bring.
 * This entry point allocates nothing.  Its scratch (split-KV partial results
 * and an error word) is a fixed array of JL_DECODE_NOALLOC_SCRATCH_BYTES in
 * the library's device image, held by every GPU that loads the library until
 * the process exits.
 *
 *   Arguments, layouts and results are those of jl_bifocal_decode, minus the
 *   workspace.  Arguments are checked exactly as jl_bifocal_decode checks them, first;
 *   then a decode whose jl_bifocal_decode_workspace_size(...) exceeds
 *   JL_DECODE_NOALLOC_SCRATCH_BYTES is rejected with JL_ERR_WORKSPACE before
 *   any launch (jl_last_error() says how much it needed).
 *   The array's device address is looked up (cudaGetSymbolAddress) by the
 *   first call made under each CUDA context and cached by that context's
 *   unique id: a context made current through the driver API, or the primary
 *   context re-created after cudaDeviceReset, gets its own lookup.  Make the
 *   first call under a context before any stream capture.  A failed lookup
 *   returns JL_ERR_CUDA.
 *   All calls share the one array, which keeps the last call's contents; the
 *   kernels clear what must start at zero.  Calls that overlap on the GPU
 *   (different streams, or different host threads, on the same device) race
 *   on the array: serialise them.
 */
#define JL_DECODE_NOALLOC_SCRATCH_BYTES (4u << 20)

jl_status jl_bifocal_decode_noalloc(const void *q, const void *k_cache,
                                    const void *v_cache,
                                    const int32_t *seqlens, int32_t batch,
                                    int32_t cache_capacity, int32_t max_seqlen,
                                    int32_t n_q_heads, int32_t n_kv_heads,
                                    int32_t head_dim, int64_t w_pretrained,
                                    int32_t w0, double rope_theta, void *out,
                                    float *lse, jl_dtype dtype, uint32_t flags,
                                    void *stream);

/*
 * jl_bifocal_decode_noalloc_error — the kernel error word of the most recent
 * jl_bifocal_decode_noalloc call under the current context.  (An addition of
 * this library; the paper has no counterpart.)
 *
 * The decode kernels report a bounded wait that ran out (a stalled pipeline:
 * the call returns, its output is not valid) by setting bits of a word in
 * their scratch; with a caller workspace that is the workspace's first int32,
 * with jl_bifocal_decode_noalloc it lives in the library's own array, which
 * the caller cannot address.  This call enqueues one device-to-host copy of
 * that word into *error_word (a host int32; pinned memory keeps the copy
 * asynchronous) on `stream`; read it after synchronising the stream.  0 means
 * no error.  NULL error_word: JL_ERR_INVALID_ARG; a failed copy: JL_ERR_CUDA.
 */
jl_status jl_bifocal_decode_noalloc_error(int32_t *error_word, void *stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* JETLONG_H */
