// Split-KV decode kernel for Dynamic Bifocal RoPE attention (sm_100a).
//
// One generation step: the new query (standard RoPE at position i = L-1)
// attends to a standard-RoPE KV cache that is never rewritten.  Local keys
// (i - j < w0) keep the base RoPE (Jet-Long technical summary, §1 "Janela
// Local"); remote keys are scored at grouped positions through the correction
// rotation of §2 "Rotação de Correção On-the-Fly".  Because RoPE rotations
// compose additively,
//     <R(delta_i) q~, R(delta_j) k~_j> = <q~, R(delta_j - delta_i) k~_j>,
// so the kernel rotates each remote key once by the relative shift
// delta_j - delta_i = -(n_j - n_i), n(p) = p - f(p), and dots it with the
// stored query.  G is recomputed from L on the device at every step.
//
// CTA (split, kv head, sequence), 256 threads, keys [split*chunk, ...):
//  * K and V tiles of 64 keys arrive by TMA (cp.async.bulk.tensor) in a
//    3-stage shared-memory ring; thread 0 refills a stage once all eight
//    warps have released it (mbarrier with one arrival per warp).
//  * a key row of D elements is read by D/8 threads ("slot"): thread t holds
//    elements [4t, 4t+4) and [D/2+4t, D/2+4t+4), i.e. whole rotation pairs.
//    Slot s takes rows s, s+S, s+2S, ... (S = number of slots), so the
//    rotation angle advances by a fixed stride; each thread carries the
//    cos/sin of its four angles as an fp32 recurrence seeded in fp64.
//  * per slot, an online softmax (running max / sum per GQA head) over its
//    rows; the slots are merged at the end, the splits by a second kernel
//    (the LSE merge of §2 "Mesclagem ... Inclusão–Exclusão" applied to key
//    ranges).
#include <algorithm>

#include "jl_common.cuh"
#include "jl_ptx.cuh"

namespace jl {

constexpr int DEC_THREADS = 256;
constexpr int DEC_TK = 64;  // keys per tile
constexpr int DEC_NST = 3;  // ring stages (each: K tile + V tile)
constexpr float LOG2E = 1.4426950408889634f;
constexpr int DEC_ERR_TIMEOUT = 8;

template <typename T>
struct Row4;  // four consecutive row elements from shared memory, as fp32
template <>
struct Row4<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const uint8_t *p, float *x) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  }
};
template <>
struct Row4<float> {
  static __device__ __forceinline__ void load(const uint8_t *p, float *x) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
};

template <typename T>
__device__ __forceinline__ void load_q4(const T *p, float *x);
template <>
__device__ __forceinline__ void load_q4<__nv_bfloat16>(const __nv_bfloat16 *p, float *x) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
template <>
__device__ __forceinline__ void load_q4<float>(const float *p, float *x) {
  const float4 v = *reinterpret_cast<const float4 *>(p);
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}

// Sum the GS per-head partials over the TPR threads of a slot and give every
// thread of the slot all GS sums.
template <int GS, int TPR>
__device__ __forceinline__ void slot_allreduce(float (&v)[GS]) {
  if constexpr (GS == 4 && TPR >= 4) {
    // transposed butterfly: two halving exchanges, then a plain reduction,
    // then a broadcast of the four head sums
    const int t = threadIdx.x % TPR;
    const bool hi = t & (TPR / 2);
    const float s0 = hi ? v[0] : v[2], s1 = hi ? v[1] : v[3];
    float k0 = hi ? v[2] : v[0], k1 = hi ? v[3] : v[1];
    k0 += __shfl_xor_sync(0xffffffffu, s0, TPR / 2);
    k1 += __shfl_xor_sync(0xffffffffu, s1, TPR / 2);
    const bool hi2 = t & (TPR / 4);
    const float s = hi2 ? k0 : k1;
    float kk = hi2 ? k1 : k0;
    kk += __shfl_xor_sync(0xffffffffu, s, TPR / 4);
#pragma unroll
    for (int o = TPR / 8; o >= 1; o >>= 1) kk += __shfl_xor_sync(0xffffffffu, kk, o);
    // thread t now holds head 2*hi + hi2; fetch every head from its owner
    const int base = (threadIdx.x & 31) & ~(TPR - 1);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int src = base + (g >> 1) * (TPR / 2) + (g & 1) * (TPR / 4);
      v[g] = __shfl_sync(0xffffffffu, kk, src);
    }
  } else {
#pragma unroll
    for (int g = 0; g < GS; ++g)
#pragma unroll
      for (int o = TPR / 2; o >= 1; o >>= 1) v[g] += __shfl_xor_sync(0xffffffffu, v[g], o);
  }
}

struct DecodeArgs {
  const void *q;
  const int32_t *seqlens;
  int Lcap, Hq, Hkv;
  long long w_pre;
  int w0, plain, chunk, nsplit;
  int window;  // sliding-window width (0: none)
  int max_seqlen;
  float *part_o, *part_ml;
  int *err;
};

template <typename T, int D, int GS>
__global__ void __launch_bounds__(DEC_THREADS, (GS <= 4 && sizeof(T) == 2) ? 2 : 1)
decode_partial_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                      const __grid_constant__ DecodeArgs p, const __grid_constant__ InvFreq inv) {
  constexpr int TPR = D / 8;
  constexpr int SLOTS = DEC_THREADS / TPR;
  constexpr int RPS = DEC_TK / SLOTS;  // rows per slot per tile
  constexpr int HALF = D / 2;
  constexpr int ROWB = D * (int)sizeof(T);
  constexpr int TILEB = DEC_TK * ROWB;
  constexpr int STAGEB = 2 * TILEB;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[DEC_NST], empty[DEC_NST];
  __shared__ volatile int abort_flag;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, slot = tid / TPR, t = tid % TPR;
  int L = p.seqlens[b];
  // a length outside [0, min(Lcap, max_seqlen)], or with more keys than the
  // planned splits hold, attends to nothing rather than reading past the
  // cache; a sliding-window layer sees keys jw .. L-1 only
  if (L < 0 || L > p.Lcap || L > p.max_seqlen) L = 0;
  int jw = p.window > 0 ? max(0, L - p.window) : 0;
  if (L - jw > p.nsplit * p.chunk) L = jw = 0;
  const int kb = jw + split * p.chunk;
  const int ke = min(L, kb + p.chunk);
  const int n = max(0, ke - kb);
  const size_t pidx = ((size_t)b * p.Hq + (size_t)kvh * GS) * p.nsplit + split;  // + g * nsplit

  if (n == 0) {  // nothing to attend in this split
    for (int idx = tid; idx < GS * D; idx += DEC_THREADS)
      p.part_o[(pidx + (size_t)(idx / D) * p.nsplit) * D + idx % D] = 0.f;
    if (tid < GS) {
      p.part_ml[(pidx + (size_t)tid * p.nsplit) * 2 + 0] = -INFINITY;
      p.part_ml[(pidx + (size_t)tid * p.nsplit) * 2 + 1] = 0.f;
    }
    return;
  }
  const int ntiles = (n + DEC_TK - 1) / DEC_TK;
  const int row0 = b * p.Lcap + kb;  // cache row of this split's first key
  const uint32_t sbase = su32(smem);

  if (tid == 0) {
    for (int s = 0; s < DEC_NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DEC_THREADS / 32);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int issued = 0;  // tiles whose loads thread 0 has issued
  if (tid == 0) {
    for (int u = 0; u < min(DEC_NST, ntiles); ++u, ++issued) {
      mbar_expect_tx(&full[u], STAGEB);
      tma_load(&mK, &full[u], sbase + u * STAGEB, 0, kvh, row0 + u * DEC_TK);
      tma_load(&mV, &full[u], sbase + u * STAGEB + TILEB, 0, kvh, row0 + u * DEC_TK);
    }
  }

  const int i = L - 1;  // query position
  const int G = p.plain ? 1 : (int)group_size(L, p.w_pre);
  const bool bif = G > 1;
  const int j_local = (int)max(0LL, (long long)L - (long long)p.w0);  // keys >= j_local are local
  const float sl2 = rsqrtf((float)D) * LOG2E;

  float qv[GS][8];
#pragma unroll
  for (int g = 0; g < GS; ++g) {
    const T *qp = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + (size_t)kvh * GS + g) * D;
    load_q4<T>(qp + 4 * t, &qv[g][0]);
    load_q4<T>(qp + HALF + 4 * t, &qv[g][4]);
  }

  // rotation state for this slot's current key j: cos/sin((n_j - n_i) w_k),
  // advanced by SLOTS positions per row
  float ec[4], es[4], w1c[4], w1s[4], w0c[4], w0s[4];
  int rm = 0;
  const int stride_full = SLOTS - SLOTS / max(G, 1);  // n advance without a carry
  const int smod = SLOTS % max(G, 1);
  if (bif) {
    const int jf = kb + slot;
    const int ni = corr_n(i, G);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const double w = inv.v[4 * t + q4];
      angle_cs(corr_n(jf, G) - ni, w, ec[q4], es[q4]);
      angle_cs(stride_full, w, w1c[q4], w1s[q4]);
      angle_cs(stride_full - 1, w, w0c[q4], w0s[q4]);
    }
    rm = jf % G;
  }

  float m_run[GS], l_run[GS], o[GS][8];
#pragma unroll
  for (int g = 0; g < GS; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[g][e] = 0.f;
  }

  bool ok = true;
  for (int u = 0; u < ntiles; ++u) {
    const int st = u % DEC_NST;
    ok = __all_sync(0xffffffffu, wait_b(&full[st], (u / DEC_NST) & 1, &abort_flag, p.err, DEC_ERR_TIMEOUT));
    if (!ok) break;
    const uint8_t *kt = smem + st * STAGEB;
    const uint8_t *vt = kt + TILEB;
    const int j0 = kb + u * DEC_TK;
    float sc[RPS][GS];
#pragma unroll
    for (int m = 0; m < RPS; ++m) {
      const int r = slot + m * SLOTS;
      const int j = j0 + r;
      float kx[8];
      Row4<T>::load(kt + r * ROWB + 4 * t * (int)sizeof(T), &kx[0]);
      Row4<T>::load(kt + r * ROWB + (HALF + 4 * t) * (int)sizeof(T), &kx[4]);
      if (bif && j < j_local) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) rot_back(kx[q4], kx[4 + q4], ec[q4], es[q4]);
      }
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qv[g][e], kx[e], a);
        sc[m][g] = a;
      }
      slot_allreduce<GS, TPR>(sc[m]);
      const bool valid = j < ke;
#pragma unroll
      for (int g = 0; g < GS; ++g) sc[m][g] = valid ? sc[m][g] * sl2 : -INFINITY;
      if (bif) {  // advance j -> j + SLOTS: n grows by SLOTS - floor((j+SLOTS)/G) + floor(j/G)
        rm += smod;
        const bool carry = rm >= G;
        if (carry) rm -= G;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float wc = carry ? w0c[q4] : w1c[q4];
          const float ws = carry ? w0s[q4] : w1s[q4];
          const float c2 = ec[q4] * wc - es[q4] * ws;
          const float s2 = es[q4] * wc + ec[q4] * ws;
          ec[q4] = c2;
          es[q4] = s2;
        }
      }
    }
    // online softmax over this slot's rows of the tile
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      float mt = sc[0][g];
#pragma unroll
      for (int m = 1; m < RPS; ++m) mt = fmaxf(mt, sc[m][g]);
      if (mt > m_run[g]) {
        const float f = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - mt);
        l_run[g] *= f;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[g][e] *= f;
        m_run[g] = mt;
      }
    }
#pragma unroll
    for (int m = 0; m < RPS; ++m) {
      const int r = slot + m * SLOTS;
      if (j0 + r >= ke) continue;  // past the last key: the cache may hold anything there
      float vx[8];
      Row4<T>::load(vt + r * ROWB + 4 * t * (int)sizeof(T), &vx[0]);
      Row4<T>::load(vt + r * ROWB + (HALF + 4 * t) * (int)sizeof(T), &vx[4]);
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        const float pr = (sc[m][g] == -INFINITY) ? 0.f : exp2f(sc[m][g] - m_run[g]);
        l_run[g] += pr;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[g][e] = fmaf(pr, vx[e], o[g][e]);
      }
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&empty[st]);
    if (tid == 0 && u + DEC_NST < ntiles) {
      // refill this stage once every warp has released it
      if (!wait_b(&empty[st], (u / DEC_NST) & 1, &abort_flag, p.err, DEC_ERR_TIMEOUT)) {
        ok = false;
      } else {
        const int un = u + DEC_NST;
        mbar_expect_tx(&full[st], STAGEB);
        tma_load(&mK, &full[st], sbase + st * STAGEB, 0, kvh, row0 + un * DEC_TK);
        tma_load(&mV, &full[st], sbase + st * STAGEB + TILEB, 0, kvh, row0 + un * DEC_TK);
        ++issued;
      }
    }
  }
  // every load issued must land before the shared memory is reused or freed
  if (tid == 0) {
    for (int u = max(0, issued - DEC_NST); u < issued; ++u) {
      // the last load of each stage is tile u (those before it were consumed)
      wait_drain(&full[u % DEC_NST], (u / DEC_NST) & 1, p.err, DEC_ERR_TIMEOUT);
    }
  }
  __syncthreads();

  // ---- merge the slots: (m, l, O) per head -> this split's partial
  float *red_o = reinterpret_cast<float *>(smem);          // [SLOTS][GS][D]
  float *red_m = red_o + SLOTS * GS * D;                    // [SLOTS][GS]
  float *red_l = red_m + SLOTS * GS;                        // [SLOTS][GS]
#pragma unroll
  for (int g = 0; g < GS; ++g) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int d = (e < 4) ? (4 * t + e) : (HALF + 4 * t + e - 4);
      red_o[(slot * GS + g) * D + d] = o[g][e];
    }
    if (t == 0) {
      red_m[slot * GS + g] = m_run[g];
      red_l[slot * GS + g] = l_run[g];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < GS * D; idx += DEC_THREADS) {
    const int g = idx / D, d = idx % D;
    float M = -INFINITY;
    for (int s = 0; s < SLOTS; ++s) M = fmaxf(M, red_m[s * GS + g]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY && ok) {
      for (int s = 0; s < SLOTS; ++s) {
        const float ms = red_m[s * GS + g];
        if (ms == -INFINITY) continue;
        const float w = exp2f(ms - M);
        acc = fmaf(w, red_o[(s * GS + g) * D + d], acc);
        lsum = fmaf(w, red_l[s * GS + g], lsum);
      }
    } else {
      M = -INFINITY;
    }
    p.part_o[(pidx + (size_t)g * p.nsplit) * D + d] = acc;
    if (d == 0) {
      p.part_ml[(pidx + (size_t)g * p.nsplit) * 2 + 0] = M;
      p.part_ml[(pidx + (size_t)g * p.nsplit) * 2 + 1] = lsum;
    }
  }
}

// LSE-weighted merge of the splits of one (sequence, query head).
template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml, int nsplit,
                      const int2 *__restrict__ plan_tab, int GS, int Hkv, T *__restrict__ out,
                      float *__restrict__ lse) {
  const int bh = blockIdx.x, d = threadIdx.x;
  // rows of this (sequence, head)'s splits: row0 + s * stride, s < ns.  With
  // a balanced plan the rows are per unit (GS heads each) and the plan's
  // table gives the sequence's first unit and units per kv head.
  size_t row0 = (size_t)bh * nsplit, stride = 1;
  int ns = nsplit;
  if (plan_tab != nullptr) {
    const int Hq = GS * Hkv, b = bh / Hq, h = bh % Hq;
    const int2 e = plan_tab[b];
    ns = e.y;
    row0 = ((size_t)e.x + (size_t)(h / GS) * ns) * GS + h % GS;
    stride = GS;
  }
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, part_ml[(row0 + s * stride) * 2]);
  float acc = 0.f, l = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const size_t row = row0 + s * stride;
      const float m = part_ml[row * 2];
      if (m == -INFINITY) continue;
      const float w = exp2f(m - M);
      l = fmaf(w, part_ml[row * 2 + 1], l);
      acc = fmaf(w, part_o[row * D + d], acc);
    }
  }
  out[(size_t)bh * D + d] = from_f<T>(l > 0.f ? acc / l : 0.f);
  if (lse != nullptr && d == 0) lse[bh] = l > 0.f ? (M + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------

struct DecodePlan {
  int nsplit;
  int chunk;
  size_t smem_bytes;
};

static size_t decode_smem(int elem, int D, int GS) {
  const int tpr = D / 8, slots = DEC_THREADS / tpr;
  const size_t ring = (size_t)DEC_NST * 2 * DEC_TK * D * elem;
  const size_t red = (size_t)slots * GS * (D + 2) * sizeof(float);
  return ring > red ? ring : red;
}

// (sequence, kv head) pairs of a call, at least 1; computed in 64 bits and
// clamped, since batch and Hkv may each be up to 65535
static int sequence_heads(int batch, int Hkv) {
  const long long bh = (long long)batch * (long long)Hkv;
  return bh < 1 ? 1 : (bh > INT32_MAX ? INT32_MAX : (int)bh);
}

// Split count: one wave of CTAs (148 SMs x CTAs resident per SM), splits of at
// least one 64-key tile, rounded to whole tiles.
DecodePlan decode_plan(int batch, int Hq, int Hkv, int D, int max_seqlen, int elem) {
  DecodePlan p;
  const int GS = Hq / Hkv;
  const int per_sm = (GS <= 4 && elem == 2) ? 2 : 1;
  const int target = 148 * per_sm;
  const int per_bh = sequence_heads(batch, Hkv);
  int ns = max(1, target / per_bh);
  const int maxL = max(1, max_seqlen);
  int chunk = (maxL + ns - 1) / ns;
  chunk = (chunk + DEC_TK - 1) / DEC_TK * DEC_TK;
  ns = (maxL + chunk - 1) / chunk;
  p.nsplit = ns;
  p.chunk = chunk;
  p.smem_bytes = decode_smem(elem, D, GS);
  return p;
}

static bool make_cache_map(CUtensorMap *m, const void *base, int rows, int Hkv, int D, int elem) {
  EncodeTiledFn enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * elem, (cuuint64_t)Hkv * D * elem};
  cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)DEC_TK};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int GS>
static cudaError_t launch_decode_t(const CUtensorMap &mK, const CUtensorMap &mV, const DecodeArgs &a,
                                   const InvFreq &inv, int B, const DecodePlan &pl, void *out, float *lse,
                                   cudaStream_t st) {
  auto kern = decode_partial_kernel<T, D, GS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(pl.nsplit, a.Hkv, B);
  kern<<<grid, DEC_THREADS, pl.smem_bytes, st>>>(mK, mV, a, inv);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  decode_combine_kernel<T, D><<<B * a.Hq, D, 0, st>>>(a.part_o, a.part_ml, pl.nsplit, nullptr, 1, 1, (T *)out,
                                                      lse);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_decode_d(int GS, const CUtensorMap &mK, const CUtensorMap &mV, const DecodeArgs &a,
                                   const InvFreq &inv, int B, const DecodePlan &pl, void *out, float *lse,
                                   cudaStream_t st) {
  switch (GS) {
    case 1: return launch_decode_t<T, D, 1>(mK, mV, a, inv, B, pl, out, lse, st);
    case 2: return launch_decode_t<T, D, 2>(mK, mV, a, inv, B, pl, out, lse, st);
    case 4: return launch_decode_t<T, D, 4>(mK, mV, a, inv, B, pl, out, lse, st);
    case 8: return launch_decode_t<T, D, 8>(mK, mV, a, inv, B, pl, out, lse, st);
  }
  return cudaErrorInvalidValue;
}

void decode_tc_plan(int batch, int Hkv, int D, int max_seqlen, int *nsplit, int *chunk);
cudaError_t launch_decode_tc(int GS, int D, const CUtensorMap &mK, const CUtensorMap &mV, const __nv_bfloat16 *q,
                             const int32_t *seqlens, int B, int Lcap, int max_seqlen, int Hq, int Hkv,
                             long long w_pre, int w0, int window, const InvFreq &inv, int plain, int nsplit,
                             int chunk, float *part_o, float *part_ml, int2 *plan_tab, __nv_bfloat16 *out,
                             float *lse, int *err, cudaStream_t st);

static bool use_tc_decode(bool bf16, int D, int GS) { return bf16 && (D == 128 || D == 64) && GS <= 8; }

// Rows of split partials the workspace must hold: a bound on the split count
// of every plan either decode kernel may use for any key count up to
// max_seqlen (a sliding window plans over fewer keys).  A plan never has more
// splits than its per-(sequence, kv head) share of a wave, nor more than one
// per key tile.
size_t decode_partial_rows(int batch, int Hq, int Hkv, int D, int max_seqlen) {
  const int GS = Hq / Hkv;
  const int per_bh = sequence_heads(batch, Hkv);
  const int tiles64 = (max(1, max_seqlen) + DEC_TK - 1) / DEC_TK;
  int ns = min(max(1, 2 * 148 / per_bh), tiles64);  // both element sizes of decode_plan
  if (use_tc_decode(true, D, GS)) ns = max(ns, min(max(1, 148 / per_bh), (max(1, max_seqlen) + 127) / 128));
  size_t rows = (size_t)batch * Hq * ns;
  // the tensor-core decode's balanced plan: at most one unit of GS rows per SM
  if (use_tc_decode(true, D, GS) && per_bh < 148) rows = std::max(rows, (size_t)148 * GS);
  return rows;
}

// Whether the tensor-core decode plans its splits on the device: for two or
// more sequences (whose lengths may differ) in fewer (sequence, kv head)
// pairs than SMs.  A single sequence keeps the host plan, sized by
// max_seqlen: the device plan costs ~2 us per step, which only pays when
// lengths differ (or the one length is well below max_seqlen).  Also the
// bytes of the plan's table.
static bool decode_tc_balanced(int batch, int Hkv) { return batch >= 2 && sequence_heads(batch, Hkv) < 148; }
size_t decode_plan_tab_bytes() { return 148 * sizeof(int2); }

static bool make_tile_map(CUtensorMap *m, const void *base, int rows, int Hkv, int D) {
  // bf16 cache viewed as (d, head, row); 64 x 1 x (keys of a tile) boxes,
  // 128-byte swizzle: 128 keys at head_dim 128, 256 at 64
  EncodeTiledFn enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, D == 64 ? 256u : 128u};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_decode(bool bf16, int D, int GS, const void *q, const void *kc, const void *vc,
                          const int32_t *seqlens, int B, int Lcap, int max_seqlen, int Hq, int Hkv,
                          long long w_pre, int w0, int window, const InvFreq &inv, int plain, float *part_o,
                          float *part_ml, int2 *plan_tab, int *err, void *out, float *lse, cudaStream_t st) {
  const int elem = bf16 ? 2 : 4;
  // the splits cover at most `window` keys per sequence
  const int keys = window > 0 ? min(max_seqlen, window) : max_seqlen;
  if (use_tc_decode(bf16, D, GS)) {
    CUtensorMap tK, tV;
    if (!make_tile_map(&tK, kc, B * Lcap, Hkv, D) || !make_tile_map(&tV, vc, B * Lcap, Hkv, D))
      return cudaErrorInvalidValue;
    int ns, chunk;
    decode_tc_plan(B, Hkv, D, keys, &ns, &chunk);
    int2 *tab = decode_tc_balanced(B, Hkv) ? plan_tab : nullptr;
    cudaError_t e = launch_decode_tc(GS, D, tK, tV, (const __nv_bfloat16 *)q, seqlens, B, Lcap, max_seqlen, Hq, Hkv,
                                     w_pre, w0, window, inv, plain, ns, chunk, part_o, part_ml, tab,
                                     (__nv_bfloat16 *)out, lse, err, st);
    if (e != cudaSuccess) return e;
    if (D == 128)
      decode_combine_kernel<__nv_bfloat16, 128><<<B * Hq, 128, 0, st>>>(part_o, part_ml, ns, tab, GS, Hkv,
                                                                        (__nv_bfloat16 *)out, lse);
    else
      decode_combine_kernel<__nv_bfloat16, 64><<<B * Hq, 64, 0, st>>>(part_o, part_ml, ns, tab, GS, Hkv,
                                                                      (__nv_bfloat16 *)out, lse);
    return cudaGetLastError();
  }
  const DecodePlan pl = decode_plan(B, Hq, Hkv, D, keys, elem);
  CUtensorMap mK, mV;
  if (!make_cache_map(&mK, kc, B * Lcap, Hkv, D, elem) || !make_cache_map(&mV, vc, B * Lcap, Hkv, D, elem))
    return cudaErrorInvalidValue;
  DecodeArgs a;
  a.q = q;
  a.seqlens = seqlens;
  a.Lcap = Lcap;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.w_pre = w_pre;
  a.w0 = w0;
  a.plain = plain;
  a.window = window;
  a.max_seqlen = max_seqlen;
  a.chunk = pl.chunk;
  a.nsplit = pl.nsplit;
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.err = err;
  if (bf16) {
    if (D == 128) return launch_decode_d<__nv_bfloat16, 128>(GS, mK, mV, a, inv, B, pl, out, lse, st);
    if (D == 64) return launch_decode_d<__nv_bfloat16, 64>(GS, mK, mV, a, inv, B, pl, out, lse, st);
  } else {
    if (D == 128) return launch_decode_d<float, 128>(GS, mK, mV, a, inv, B, pl, out, lse, st);
    if (D == 64) return launch_decode_d<float, 64>(GS, mK, mV, a, inv, B, pl, out, lse, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace jl

// ---------------------------------------------------------------------------
// Allocation-free decode entry point
//
// Some callers cannot call cudaMalloc: a plugin hosted by a runtime that owns
// the whole device-memory budget (its allocator hands out nothing outside its
// own pools), or a latency-critical generation loop that must not risk the
// implicit device synchronisation an allocation can cause.  For them
// jl_bifocal_decode_noalloc runs the same split-KV decode with its scratch
// (the per-split partial results and an error word) in a fixed array that
// lives in the library's own device image.
// ---------------------------------------------------------------------------
#include <mutex>

#include "../../include/jetlong.h"

namespace jl {
void set_last_error(const char *fmt, ...);
}

// File-scope scratch of JL_DECODE_NOALLOC_SCRATCH_BYTES.  Every GPU that loads
// the library holds it until the process exits.  In host code this name is
// only a host-side stand-in: the device address comes from
// cudaGetSymbolAddress, looked up below once per CUDA context.
static __device__ __align__(256) uint8_t g_decode_scratch[JL_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

std::mutex g_scratch_mu;
// The symbol's address belongs to the context (module instance) that was
// current when it was looked up: a driver-API context made current by a host
// runtime, or the primary context re-created after cudaDeviceReset, has its
// own.  So the cache is keyed by the context's unique id, which a new context
// never shares with an old one.
struct ScratchEntry {
  unsigned long long ctx_id;
  void *addr;
};
ScratchEntry g_scratch_cache[64];
int g_scratch_n = 0;

template <typename Fn>
Fn driver_fn(const char *name) {
  void *ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(ptr);
}

// Unique id of the context current on this thread (0 if none is current yet).
cudaError_t current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (get_cur == nullptr || get_id == nullptr) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  *id = 0;
  if (ctx != nullptr && get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  return cudaSuccess;
}

// Device address of g_decode_scratch in the context current on this thread.
// The first call under a context looks it up (which also makes the runtime's
// primary context current when none was); later calls find it in the cache.
cudaError_t scratch_for_current_context(void **out) {
  unsigned long long id = 0;
  cudaError_t e = current_context_id(&id);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  for (int i = 0; i < g_scratch_n; ++i)
    if (id != 0 && g_scratch_cache[i].ctx_id == id) {
      *out = g_scratch_cache[i].addr;
      return cudaSuccess;
    }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  if (id == 0 && (e = current_context_id(&id)) != cudaSuccess) return e;  // the lookup made one current
  if (id != 0) {
    // keep the newest 64 contexts; an evicted one only costs a new lookup
    const int slot = g_scratch_n < 64 ? g_scratch_n++ : (int)(id % 64);
    g_scratch_cache[slot] = ScratchEntry{id, p};
  }
  *out = p;
  return cudaSuccess;
}
}  // namespace

extern "C" jl_status jl_bifocal_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                               const int32_t *seqlens, int32_t batch, int32_t cache_capacity,
                                               int32_t max_seqlen, int32_t n_q_heads, int32_t n_kv_heads,
                                               int32_t head_dim, int64_t w_pretrained, int32_t w0,
                                               double rope_theta, void *out, float *lse, jl_dtype dtype,
                                               uint32_t flags, void *stream) {
  // Argument checks first, exactly those of jl_bifocal_decode: a dry run with
  // an impossible (NULL) workspace returns every argument error, and
  // JL_ERR_WORKSPACE only once the arguments are valid.
  jl_status s = jl_bifocal_decode(q, k_cache, v_cache, seqlens, batch, cache_capacity, max_seqlen, n_q_heads,
                                  n_kv_heads, head_dim, w_pretrained, w0, rope_theta, out, lse, nullptr, 0, dtype,
                                  flags, stream);
  if (s != JL_ERR_WORKSPACE) return s;  // an argument error, or JL_OK for an empty batch
  const size_t need = jl_bifocal_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_seqlen);
  if (need > (size_t)JL_DECODE_NOALLOC_SCRATCH_BYTES) {
    jl::set_last_error("this decode needs %zu bytes of scratch; the allocation-free entry point has a fixed %u "
                       "bytes (use jl_bifocal_decode with a caller workspace)",
                       need, (unsigned)JL_DECODE_NOALLOC_SCRATCH_BYTES);
    return JL_ERR_WORKSPACE;
  }
  void *scratch = nullptr;
  const cudaError_t e = scratch_for_current_context(&scratch);
  if (e != cudaSuccess) {
    jl::set_last_error("looking up the decode scratch address failed: %s", cudaGetErrorString(e));
    return JL_ERR_CUDA;
  }
  return jl_bifocal_decode(q, k_cache, v_cache, seqlens, batch, cache_capacity, max_seqlen, n_q_heads, n_kv_heads,
                           head_dim, w_pretrained, w0, rope_theta, out, lse, scratch,
                           (size_t)JL_DECODE_NOALLOC_SCRATCH_BYTES, dtype, flags, stream);
}

extern "C" jl_status jl_bifocal_decode_noalloc_error(int32_t *error_word, void *stream) {
  if (error_word == nullptr) {
    jl::set_last_error("error_word is NULL");
    return JL_ERR_INVALID_ARG;
  }
  void *scratch = nullptr;
  cudaError_t e = scratch_for_current_context(&scratch);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(error_word, scratch, sizeof(int32_t), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    jl::set_last_error("reading the decode scratch error word failed: %s", cudaGetErrorString(e));
    return JL_ERR_CUDA;
  }
  return JL_OK;
}

// Host copy of the decode split plan, for tests: the plan launch_decode uses
// for these sizes (tensor-core kernel for bf16 at head_dim 64 / 128 with a
// GQA group <= 8, the CUDA-core kernel otherwise) and the partial rows the
// workspace holds.  Returns 0, or -1 for sizes outside the decode's range.
extern "C" int jl_debug_decode_plan(int batch, int Hq, int Hkv, int D, int max_seqlen, int window, int bf16,
                                    int *nsplit, int *chunk, long long *partial_rows) {
  if (batch < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (D != 64 && D != 128) || max_seqlen < 1 ||
      window < 0 || nsplit == nullptr || chunk == nullptr || partial_rows == nullptr)
    return -1;
  const int GS = Hq / Hkv;
  const int keys = window > 0 ? min(max_seqlen, window) : max_seqlen;
  if (jl::use_tc_decode(bf16 != 0, D, GS)) {
    jl::decode_tc_plan(batch, Hkv, D, keys, nsplit, chunk);
  } else {
    const jl::DecodePlan pl = jl::decode_plan(batch, Hq, Hkv, D, keys, bf16 ? 2 : 4);
    *nsplit = pl.nsplit;
    *chunk = pl.chunk;
  }
  *partial_rows = (long long)jl::decode_partial_rows(batch, Hq, Hkv, D, max_seqlen);
  return 0;
}

namespace jl {
// Test hook: the limit of the bounded waits of this file's kernels.
cudaError_t set_wait_limit_decode(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}
}  // namespace jl
