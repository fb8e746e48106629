// Split-KV decode kernel for Dynamic Bifocal RoPE attention.
//
// One generation step: the new query (standard RoPE at position L-1) attends
// to a standard-RoPE KV cache that is never rewritten.  Remote keys
// (L-1 - j >= w0) are re-phased on the fly into grouped positions with the
// correction rotation R(f(j) - j), the query with R(f(L-1) - (L-1))
// (Jet-Long technical summary, §2 "Rotação de Correção On-the-Fly"); local
// keys keep the base RoPE (§1 "Janela Local").  G is recomputed from L on the
// device at every step.
//
// Work split: CTA (split, kv head, sequence) owns keys [split*chunk, ...).
//  pass 1  streams K rows with coalesced 8-byte loads: a key row of D bf16 is
//          read by D/8 threads, thread t holding elements [4t, 4t+4) and
//          [D/2 + 4t, D/2 + 4t + 4) so that each rotation pair (x_k, x_{k+D/2})
//          lives in one thread.  The rotation angle n(j) * w_k with
//          n(j) = j - f(j) advances by one position or none from key to key,
//          so each thread carries cos/sin of its four angles as an fp32
//          recurrence seeded exactly (fp64) at the start of its key range.
//          The GQA group's scores are reduced across the row's threads with a
//          transposed butterfly and kept in shared memory.
//  pass 2  takes the per-head max, exponentiates in shared memory and
//          streams V rows the same way, accumulating O per head.
//  combine merges the splits with their (max, sum) statistics (the LSE merge).
#include "jl_common.cuh"

namespace jl {

constexpr int DEC_THREADS = 128;
constexpr int DEC_UNROLL = 4;
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ void unpack4(uint2 u, float *x) {
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
}

__device__ __forceinline__ uint2 ld_stream8(const void *p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

template <typename T>
struct Row4;  // four consecutive elements of a row
template <>
struct Row4<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *x) { unpack4(ld_stream8(p), x); }
};
template <>
struct Row4<float> {
  static __device__ __forceinline__ void load(const float *p, float *x) {
    float4 v = __ldg(reinterpret_cast<const float4 *>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
};

// Sum of GS per-head partials over the TPR threads of one key row.  On return
// `out` is the full score of head `head` (valid in threads whose lowest
// bits are zero, see `owner`).
template <int GS, int TPR>
__device__ __forceinline__ void reduce_heads(const float (&v)[GS], int t, float &out, int &head,
                                             bool &owner) {
  if constexpr (GS == 4 && TPR >= 4) {
    const bool hi = t & (TPR / 2);
    float s0 = hi ? v[0] : v[2], s1 = hi ? v[1] : v[3];
    float k0 = hi ? v[2] : v[0], k1 = hi ? v[3] : v[1];
    k0 += __shfl_xor_sync(0xffffffffu, s0, TPR / 2);
    k1 += __shfl_xor_sync(0xffffffffu, s1, TPR / 2);
    const bool hi2 = t & (TPR / 4);
    float s = hi2 ? k0 : k1;
    float kk = hi2 ? k1 : k0;
    kk += __shfl_xor_sync(0xffffffffu, s, TPR / 4);
#pragma unroll
    for (int o = TPR / 8; o >= 1; o >>= 1) kk += __shfl_xor_sync(0xffffffffu, kk, o);
    out = kk;
    head = 2 * (hi ? 1 : 0) + (hi2 ? 1 : 0);
    owner = (t & (TPR / 4 - 1)) == 0;
  } else {
    float acc[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      acc[g] = v[g];
#pragma unroll
      for (int o = TPR / 2; o >= 1; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o);
    }
    // thread t < GS reports head t
    out = acc[0];
#pragma unroll
    for (int g = 1; g < GS; ++g)
      if (t == g) out = acc[g];
    head = t;
    owner = t < GS;
  }
}

template <typename T, int D, int GS>
__global__ void __launch_bounds__(DEC_THREADS)
decode_partial_kernel(const T *__restrict__ q, const T *__restrict__ kc, const T *__restrict__ vc,
                      const int32_t *__restrict__ seqlens, int Lcap, int Hq, int Hkv,
                      long long w_pre, int w0, InvFreq inv, int plain, int chunk, int nsplit,
                      float *__restrict__ part_o, float *__restrict__ part_ml) {
  constexpr int TPR = D / 8;                 // threads per key row
  constexpr int SLOTS = DEC_THREADS / TPR;   // key rows in flight per step
  constexpr int HALF = D / 2;
  extern __shared__ float smem[];            // scores [chunk][GS]; later the O reduction
  __shared__ float head_m[GS], head_l[GS];
  __shared__ float warp_red[DEC_THREADS / 32][GS];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, slot = tid / TPR, t = tid % TPR;
  int L = seqlens[b];
  // a length outside [0, min(Lcap, nsplit * chunk)] attends to nothing rather
  // than reading past the cache
  if (L < 0 || L > Lcap || L > nsplit * chunk) L = 0;
  const int kb = split * chunk;
  const int ke = min(L, kb + chunk);
  const int n = max(0, ke - kb);
  const size_t pidx = ((size_t)b * Hq + (size_t)kvh * GS) * nsplit + split;  // head g adds g*nsplit

  if (n == 0) {  // nothing to attend in this split
    for (int idx = tid; idx < GS * D; idx += DEC_THREADS) {
      const int g = idx / D, e = idx % D;
      part_o[(pidx + (size_t)g * nsplit) * D + e] = 0.f;
    }
    if (tid < GS) {
      part_ml[(pidx + (size_t)tid * nsplit) * 2 + 0] = -INFINITY;
      part_ml[(pidx + (size_t)tid * nsplit) * 2 + 1] = 0.f;
    }
    return;
  }

  const int i = L - 1;                                   // query position
  const int G = plain ? 1 : (int)group_size(L, w_pre);
  const bool bif = G > 1;
  const int j_local = (int)max(0LL, (long long)L - (long long)w0);  // keys >= j_local are local
  const float sc = rsqrtf((float)D) * LOG2E;             // scores kept in log2 units

  // ---- query: base and corrected copies of this thread's 8 elements per head
  float qs[GS][8], qg[GS][8];
#pragma unroll
  for (int g = 0; g < GS; ++g) {
    const T *qp = q + ((size_t)b * Hq + (size_t)kvh * GS + g) * D;
    Row4<T>::load(qp + 4 * t, &qs[g][0]);
    Row4<T>::load(qp + HALF + 4 * t, &qs[g][4]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qg[g][e] = qs[g][e];
  }
  if (bif && i - 0 >= w0) {
    const int ni = corr_n(i, G);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float c, s;
      angle_cs(ni, inv.v[4 * t + p], c, s);
#pragma unroll
      for (int g = 0; g < GS; ++g) rot_back(qg[g][p], qg[g][4 + p], c, s);
    }
  }

  // ---- per-slot contiguous key range, identical trip count for all slots
  const int per = (n + SLOTS - 1) / SLOTS;
  const int per_u = (per + DEC_UNROLL - 1) / DEC_UNROLL * DEC_UNROLL;
  const int js = kb + slot * per;
  const int je = min(ke, js + per);

  // rotation recurrence state: cos/sin(n(j) w_k) for the slot's current key j
  float ec[4], es[4], wc[4], ws[4];
  int cnt = 0;  // (j + 1) % G
  if (bif) {
    const int n0 = corr_n(max(js, 0), G);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      angle_cs(n0, inv.v[4 * t + p], ec[p], es[p]);
      angle_cs(1, inv.v[4 * t + p], wc[p], ws[p]);
    }
    cnt = (js + 1) % G;
  }

  const size_t row_stride = (size_t)Hkv * D;
  const T *kbase = kc + ((size_t)b * Lcap) * row_stride + (size_t)kvh * D;
  const T *vbase = vc + ((size_t)b * Lcap) * row_stride + (size_t)kvh * D;

  // ---- pass 1: scores
  for (int u0 = 0; u0 < per_u; u0 += DEC_UNROLL) {
    float kx[DEC_UNROLL][8];
#pragma unroll
    for (int u = 0; u < DEC_UNROLL; ++u) {
      const int j = js + u0 + u;
      if (j < je) {
        const T *kp = kbase + (size_t)j * row_stride;
        Row4<T>::load(kp + 4 * t, &kx[u][0]);
        Row4<T>::load(kp + HALF + 4 * t, &kx[u][4]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) kx[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < DEC_UNROLL; ++u) {
      const int j = js + u0 + u;
      const bool remote = bif && j < j_local;
      float part[GS];
      if (remote) {
#pragma unroll
        for (int p = 0; p < 4; ++p) rot_back(kx[u][p], kx[u][4 + p], ec[p], es[p]);
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(qg[g][e], kx[u][e], a);
          part[g] = a;
        }
      } else {
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(qs[g][e], kx[u][e], a);
          part[g] = a;
        }
      }
      float sres;
      int head;
      bool owner;
      reduce_heads<GS, TPR>(part, t, sres, head, owner);
      if (owner && j < je) smem[(j - kb) * GS + head] = sres * sc;
      if (bif) {  // advance n(j) -> n(j+1): +1 unless j+1 starts a new group
        const bool step = cnt != 0;
        cnt = (cnt + 1 == G) ? 0 : cnt + 1;
        if (step) {
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float c2 = ec[p] * wc[p] - es[p] * ws[p];
            const float s2 = es[p] * wc[p] + ec[p] * ws[p];
            ec[p] = c2;
            es[p] = s2;
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- per-head max and exponentials over this split's scores
  {
    float mx[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) mx[g] = -INFINITY;
    for (int r = tid; r < n; r += DEC_THREADS)
#pragma unroll
      for (int g = 0; g < GS; ++g) mx[g] = fmaxf(mx[g], smem[r * GS + g]);
#pragma unroll
    for (int g = 0; g < GS; ++g)
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
    if ((tid & 31) == 0)
#pragma unroll
      for (int g = 0; g < GS; ++g) warp_red[tid >> 5][g] = mx[g];
    __syncthreads();
    if (tid < GS) {
      float m = warp_red[0][tid];
      for (int w = 1; w < DEC_THREADS / 32; ++w) m = fmaxf(m, warp_red[w][tid]);
      head_m[tid] = m;
    }
    __syncthreads();
    float sm[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) sm[g] = 0.f;
    for (int r = tid; r < n; r += DEC_THREADS)
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        const float p = exp2f(smem[r * GS + g] - head_m[g]);
        smem[r * GS + g] = p;
        sm[g] += p;
      }
#pragma unroll
    for (int g = 0; g < GS; ++g)
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sm[g] += __shfl_xor_sync(0xffffffffu, sm[g], o);
    __syncthreads();
    if ((tid & 31) == 0)
#pragma unroll
      for (int g = 0; g < GS; ++g) warp_red[tid >> 5][g] = sm[g];
    __syncthreads();
    if (tid < GS) {
      float l = 0.f;
      for (int w = 0; w < DEC_THREADS / 32; ++w) l += warp_red[w][tid];
      head_l[tid] = l;
    }
    __syncthreads();
  }

  // ---- pass 2: O = sum_j p_j V_j per head
  float o[GS][8];
#pragma unroll
  for (int g = 0; g < GS; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) o[g][e] = 0.f;
  for (int u0 = 0; u0 < per_u; u0 += DEC_UNROLL) {
    float vx[DEC_UNROLL][8];
#pragma unroll
    for (int u = 0; u < DEC_UNROLL; ++u) {
      const int j = js + u0 + u;
      if (j < je) {
        const T *vp = vbase + (size_t)j * row_stride;
        Row4<T>::load(vp + 4 * t, &vx[u][0]);
        Row4<T>::load(vp + HALF + 4 * t, &vx[u][4]);
      }
    }
#pragma unroll
    for (int u = 0; u < DEC_UNROLL; ++u) {
      const int j = js + u0 + u;
      if (j < je) {
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          const float p = smem[(j - kb) * GS + g];
#pragma unroll
          for (int e = 0; e < 8; ++e) o[g][e] = fmaf(p, vx[u][e], o[g][e]);
        }
      }
    }
  }
  __syncthreads();  // scores no longer needed: reuse smem for the slot reduction

  float *red = smem;  // [SLOTS][GS][D]
#pragma unroll
  for (int g = 0; g < GS; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int d = (e < 4) ? (4 * t + e) : (HALF + 4 * t + e - 4);
      red[(slot * GS + g) * D + d] = o[g][e];
    }
  __syncthreads();
  for (int idx = tid; idx < GS * D; idx += DEC_THREADS) {
    const int g = idx / D, d = idx % D;
    float a = 0.f;
#pragma unroll 4
    for (int s = 0; s < SLOTS; ++s) a += red[(s * GS + g) * D + d];
    part_o[(pidx + (size_t)g * nsplit) * D + d] = a;
  }
  if (tid < GS) {
    part_ml[(pidx + (size_t)tid * nsplit) * 2 + 0] = head_m[tid];
    part_ml[(pidx + (size_t)tid * nsplit) * 2 + 1] = head_l[tid];
  }
}

// LSE-weighted merge of the splits of one (sequence, query head).
template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml,
                      int nsplit, T *__restrict__ out, float *__restrict__ lse) {
  const int bh = blockIdx.x, d = threadIdx.x;
  const float *ml = part_ml + (size_t)bh * nsplit * 2;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, ml[2 * s]);
  float acc = 0.f, l = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float m = ml[2 * s];
      if (m == -INFINITY) continue;
      const float w = exp2f(m - M);
      l = fmaf(w, ml[2 * s + 1], l);
      acc = fmaf(w, part_o[((size_t)bh * nsplit + s) * D + d], acc);
    }
  }
  out[(size_t)bh * D + d] = from_f<T>(l > 0.f ? acc / l : 0.f);
  if (lse != nullptr && d == 0) lse[bh] = l > 0.f ? (M + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

// ---------------------------------------------------------------------------
// host launcher (called from jl_api.cu after validation)
// ---------------------------------------------------------------------------

struct DecodePlan {
  int nsplit;
  int chunk;
  size_t smem_bytes;
};

// Split count: aim at 592 CTAs (148 SMs x 4 resident 128-thread CTAs), keep a
// split at most 2048 keys and a multiple of 32 keys.
DecodePlan decode_plan(int batch, int Hq, int Hkv, int D, int max_seqlen) {
  DecodePlan p;
  const int target = 148 * 4;
  const int per_bh = max(1, batch * Hkv);
  int ns = (target + per_bh - 1) / per_bh;
  const int maxL = max(1, max_seqlen);
  int chunk = (maxL + ns - 1) / ns;
  chunk = (chunk + 31) / 32 * 32;
  if (chunk > 2048) chunk = 2048;
  ns = (maxL + chunk - 1) / chunk;
  p.nsplit = ns;
  p.chunk = chunk;
  const int GS = Hq / Hkv;
  const int slots = DEC_THREADS / (D / 8);
  const size_t a = (size_t)chunk * GS * sizeof(float);
  const size_t r = (size_t)slots * GS * D * sizeof(float);
  p.smem_bytes = a > r ? a : r;
  return p;
}

template <typename T, int D, int GS>
static cudaError_t launch_decode_t(const void *q, const void *kc, const void *vc, const int32_t *seqlens,
                                   int B, int Lcap, int Hq, int Hkv, long long w_pre, int w0,
                                   const InvFreq &inv, int plain, const DecodePlan &p, float *part_o,
                                   float *part_ml, void *out, float *lse, cudaStream_t st) {
  auto kern = decode_partial_kernel<T, D, GS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)p.smem_bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, Hkv, B);
  kern<<<grid, DEC_THREADS, p.smem_bytes, st>>>(
      (const T *)q, (const T *)kc, (const T *)vc, seqlens, Lcap, Hq, Hkv, w_pre, w0, inv, plain,
      p.chunk, p.nsplit, part_o, part_ml);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<T, D><<<B * Hq, D, 0, st>>>(part_o, part_ml, p.nsplit, (T *)out, lse);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_decode_d(int GS, const void *q, const void *kc, const void *vc,
                                   const int32_t *seqlens, int B, int Lcap, int Hq, int Hkv,
                                   long long w_pre, int w0, const InvFreq &inv, int plain,
                                   const DecodePlan &p, float *po, float *pml, void *out, float *lse,
                                   cudaStream_t st) {
  switch (GS) {
    case 1: return launch_decode_t<T, D, 1>(q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, po, pml, out, lse, st);
    case 2: return launch_decode_t<T, D, 2>(q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, po, pml, out, lse, st);
    case 4: return launch_decode_t<T, D, 4>(q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, po, pml, out, lse, st);
    case 8: return launch_decode_t<T, D, 8>(q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, po, pml, out, lse, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(bool bf16, int D, int GS, const void *q, const void *kc, const void *vc,
                          const int32_t *seqlens, int B, int Lcap, int Hq, int Hkv, long long w_pre,
                          int w0, const InvFreq &inv, int plain, const DecodePlan &p, float *part_o,
                          float *part_ml, void *out, float *lse, cudaStream_t st) {
  if (bf16) {
    if (D == 128) return launch_decode_d<__nv_bfloat16, 128>(GS, q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, part_o, part_ml, out, lse, st);
    if (D == 64) return launch_decode_d<__nv_bfloat16, 64>(GS, q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, part_o, part_ml, out, lse, st);
  } else {
    if (D == 128) return launch_decode_d<float, 128>(GS, q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, part_o, part_ml, out, lse, st);
    if (D == 64) return launch_decode_d<float, 64>(GS, q, kc, vc, seqlens, B, Lcap, Hq, Hkv, w_pre, w0, inv, plain, p, part_o, part_ml, out, lse, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace jl
