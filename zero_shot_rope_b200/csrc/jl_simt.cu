// SIMT prefill kernel for Dynamic Bifocal RoPE attention: one warp per
// (query token, query head), fp32 arithmetic throughout.  It is the product
// path for float32 inputs and a plain, direct device cross-check of the
// tensor-core kernel for bf16 inputs.
//
// Per key it takes the score the method defines directly (Jet-Long technical
// summary, §1 "Janela Local" / "Janela Remota"): base RoPE inside the window
// w0, otherwise the grouped score after the correction rotation of §2
// "Rotação de Correção On-the-Fly" applied to the query and the key; the
// single masked online softmax over those scores is the exact value of the
// §2 inclusion–exclusion merge.  A sliding-window layer (window > 0) scores
// only the keys at distance < window.
//
// Lane l holds elements l + 32c (c < D/32); the rotation pair of element
// l + 32c (c < D/64) is element l + 32(c + D/64), so pairs never cross lanes.
#include "jl_common.cuh"

namespace jl {

template <typename T, int D>
__global__ void __launch_bounds__(128)
simt_prefill_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    T *__restrict__ out, float *__restrict__ lse, const int32_t *__restrict__ cu,
                    const int32_t *__restrict__ cu_k, int batch, int T_total, int Tk, int Hq, int Hkv,
                    long long w_pre, int w0, int window, InvFreq inv, int plain) {
  constexpr int NC = D / 32;
  constexpr int NP = NC / 2;  // rotation pairs per lane
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (long long)T_total * Hq) return;
  const int h = (int)(warp % Hq);
  const int tok = (int)(warp / Hq);

  // sequence holding `tok`: the largest s with cu[s] <= tok
  int lo = 0, hi = batch;  // invariant: cu[lo] <= tok < cu[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= tok) lo = mid; else hi = mid;
  }
  const int a = cu[lo];
  const int L = cu[lo + 1] - a;  // queries of this sequence
  const int ak = cu_k[lo];
  const int Lk = cu_k[lo + 1] - ak;  // keys: the sequence's current length
  if (a < 0 || L <= 0 || a + L > T_total || tok - a >= L || Lk < L || ak < 0 || ak + Lk > Tk)
    return;  // inconsistent prefix sums
  const int i = Lk - L + (tok - a);  // the query's position
  const int G = plain ? 1 : (int)group_size(Lk, w_pre);
  const bool bif = G > 1;
  const int kvh = h / (Hq / Hkv);
  const float scale = rsqrtf((float)D);

  float qv[NC], qg[NC];
  const T *qp = q + ((size_t)tok * Hq + h) * D;
#pragma unroll
  for (int c = 0; c < NC; ++c) qg[c] = qv[c] = to_f<T>(qp[lane + 32 * c]);
  if (bif && i >= w0) {
    const int ni = corr_n(i, G);
#pragma unroll
    for (int c = 0; c < NP; ++c) {
      float cs, sn;
      angle_cs(ni, inv.v[lane + 32 * c], cs, sn);
      rot_back(qg[c], qg[c + NP], cs, sn);
    }
  }

  float m = -INFINITY, l = 0.f, acc[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) acc[c] = 0.f;
  // a sliding-window layer hides keys at distance >= window
  for (int j = window > 0 ? max(0, i - window + 1) : 0; j <= i; ++j) {
    const T *kp = k + ((size_t)(ak + j) * Hkv + kvh) * D;
    float kx[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) kx[c] = to_f<T>(kp[lane + 32 * c]);
    float part = 0.f;
    if (bif && i - j >= w0) {  // remote: grouped positions
      const int nj = corr_n(j, G);
#pragma unroll
      for (int c = 0; c < NP; ++c) {
        float cs, sn;
        angle_cs(nj, inv.v[lane + 32 * c], cs, sn);
        rot_back(kx[c], kx[c + NP], cs, sn);
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) part = fmaf(qg[c], kx[c], part);
    } else {  // local window: base RoPE
#pragma unroll
      for (int c = 0; c < NC; ++c) part = fmaf(qv[c], kx[c], part);
    }
    const float s = warp_sum(part) * scale;
    const float m_new = fmaxf(m, s);
    const float corr = expf(m - m_new);
    const float p = expf(s - m_new);
    l = fmaf(l, corr, p);
    const T *vp = v + ((size_t)(ak + j) * Hkv + kvh) * D;
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[c] = fmaf(acc[c], corr, p * to_f<T>(vp[lane + 32 * c]));
    m = m_new;
  }
  T *op = out + ((size_t)tok * Hq + h) * D;
#pragma unroll
  for (int c = 0; c < NC; ++c) op[lane + 32 * c] = from_f<T>(acc[c] / l);
  if (lse != nullptr && lane == 0) lse[(size_t)h * T_total + tok] = m + logf(l);
}

cudaError_t launch_simt_prefill(bool bf16, int D, const void *q, const void *k, const void *v, void *out,
                                float *lse, const int32_t *cu, const int32_t *cu_k, int batch, int T_total,
                                int Tk, int Hq, int Hkv, long long w_pre, int w0, int window, const InvFreq &inv,
                                int plain, cudaStream_t st) {
  const long long warps = (long long)T_total * Hq;
  if (warps == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((warps + 3) / 4);
#define JL_SIMT(TT, DD)                                                                        \
  simt_prefill_kernel<TT, DD><<<blocks, 128, 0, st>>>((const TT *)q, (const TT *)k,            \
                                                      (const TT *)v, (TT *)out, lse, cu, cu_k,  \
                                                      batch, T_total, Tk, Hq, Hkv, w_pre, w0, window, inv, plain)
  if (bf16) {
    if (D == 128) JL_SIMT(__nv_bfloat16, 128);
    else if (D == 64) JL_SIMT(__nv_bfloat16, 64);
    else return cudaErrorInvalidValue;
  } else {
    if (D == 128) JL_SIMT(float, 128);
    else if (D == 64) JL_SIMT(float, 64);
    else return cudaErrorInvalidValue;
  }
#undef JL_SIMT
  return cudaGetLastError();
}

}  // namespace jl
