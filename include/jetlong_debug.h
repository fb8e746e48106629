/*
 * jetlong_debug.h — a test hook of the library, not an attention entry point.
 *
 * jl_debug_prefill_visits — the prefill kernels' tile schedule, computed on
 * the host by the same code the kernels run: for query tile qt (rows
 * 128 qt .. of a sequence with L queries at positions Lk - L + i over keys
 * 0 .. Lk-1), every (key tile, branch, mask) visit in the order the kernels
 * process them.  The method's routing (§1 "Janela Local" / "Janela Remota"
 * of the Jet-Long technical summary: distance d < w0 scored with the base
 * RoPE, d >= w0 at grouped positions; a sliding window hides d >= window)
 * must come out as: every visible (row, key) pair claimed by exactly one
 * visit, on the right branch.
 *   G        the group size (G = 1: no grouped visits, as in plain mode)
 *   window   0: no window
 *   out      host int array, 5 ints per visit: key tile, grouped (0/1),
 *            masked (0/1), lo, hi — a masked visit keeps the columns whose
 *            distance d satisfies lo <= d <= hi, an unmasked one all 128
 *   cap      visits that fit in out
 * Returns the number of visits (which may exceed cap), or -1 for arguments
 * outside the kernels' range (L <= 0, Lk < L, w0 < 0, window < 0, G < 1, a
 * tile past L, out NULL).  Host-only; no CUDA call.
 */
#ifndef JETLONG_DEBUG_H
#define JETLONG_DEBUG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int jl_debug_prefill_visits(int L, int Lk, int w0, int window, int G, int qt, int *out, int cap);

/*
 * jl_debug_decode_plan — the decode's split plan, computed on the host by the
 * code the decode call uses: sequence b's keys max(0, L_b - window) .. L_b-1
 * (all keys when window = 0) go to splits of `chunk` keys, `nsplit` per
 * (sequence, kv head), so every length up to max_seqlen must fit in
 * nsplit * chunk keys and the workspace's `partial_rows` must hold
 * batch * Hq * nsplit.  bf16 != 0 selects the bf16 plan (tensor-core kernel
 * at head_dim 64 / 128 with a GQA group <= 8), 0 the fp32 one.  Returns 0, or
 * -1 for sizes outside the decode's range.  Host-only; no CUDA call.
 */
int jl_debug_decode_plan(int batch, int Hq, int Hkv, int D, int max_seqlen, int window, int bf16,
                         int *nsplit, int *chunk, long long *partial_rows);

/*
 * jl_debug_set_wait_limit — the time limit, in nanoseconds, of the kernels'
 * bounded pipeline waits on the current device (0 restores the default of
 * 2 s).  A wait that runs out sets a bit of the call's error word, stops the
 * kernel's other roles, lets its own copies and tensor-core work finish and
 * returns; the call's output is then not valid.  Shortening the limit lets a
 * test make such a wait run out without withholding any work: nothing faults
 * and the context stays usable.  The waits that let a CTA's own copies land
 * before it exits keep their fixed limit.  Synchronous (cudaMemcpyToSymbol);
 * returns 0, or -1 with jl_last_error() set.
 */
int jl_debug_set_wait_limit(unsigned long long ns);

/*
 * jl_debug_angle_cs — the kernels' correction angle on the host: cos and sin
 * of n * inv_freq, evaluated in fp64 by the kernels' own call-free sine and
 * cosine and rounded to fp32.  Host-only; no CUDA call.
 */
void jl_debug_angle_cs(int32_t n, double inv_freq, float *c, float *s);

#ifdef __cplusplus
}
#endif

#endif /* JETLONG_DEBUG_H */
