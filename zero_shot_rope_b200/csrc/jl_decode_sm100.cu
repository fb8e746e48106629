// Tensor-core split-KV decode kernel for Dynamic Bifocal RoPE attention
// (sm_100a, bf16, head_dim 64 or 128, up to 8 query heads per kv head).
//
// One generation step against a standard-RoPE cache that is never rewritten
// (Jet-Long technical summary, §2 "Rotação de Correção On-the-Fly"): local
// keys (L-1 - j < w0) keep the base RoPE, remote keys are scored at grouped
// positions.  Rotations compose additively, so
//     <R(delta_i) q~, R(delta_j) k~_j> = <q~, R(delta_j - delta_i) k~_j>:
// each remote key row is rotated once, by the relative shift, and the stored
// query is used unchanged.
//
// CTA (split, kv head, sequence), 448 threads, keys [jw + split*chunk, ...) in
// tiles of 128:
//   warp 12    TMA producer: K and V tiles (128 keys x 128 d, SWIZZLE_128B) in
//              two 3-stage rings.
//   warps 4-11 rotation warps: rotate the remote rows of each K tile in shared
//              memory by R(delta_j - delta_i); thread t owns one 16-byte column
//              chunk (8 pairs) of rows t/8 + 32m.  The rotation of its first
//              row advances once per tile (fp32 recurrence, fp64 seed); its
//              other rows compose that with one of two tabulated offsets, so
//              no row waits on another.  Two pairs per packed f32x2 op.
//   warp 13    TMEM allocator and single-thread tcgen05.mma issuer, per tile
//              S^T = K Q^T   (M = 128 keys, N = 16: the GQA heads, zero-padded)
//              then O^T += V^T P  (M = 128 = head_dim, N = 16, V read MN-major)
//   warps 0-3  softmax warpgroup: thread r owns key r of the tile (S^T lane r)
//              and head-dim row r of O^T; block-wide running max per head,
//              P written to shared memory as the B operand of the PV MMA, lazy
//              O rescale, the CTA's partial (m, l, O) at the end.
// The splits are merged by decode_combine_kernel (jl_decode.cu).  Every
// mbarrier wait is bounded; on expiry the kernel records an error bit in the
// workspace, stops the other roles, drains its own copies and MMAs, frees
// TMEM and returns.
#include "jl_common.cuh"
#include "jl_ptx.cuh"

namespace jl {
namespace dtc {

// keys per tile: 128 at head_dim 128; 256 at head_dim 64, so that a K or V
// stage holds 32 KB and a tile's fixed costs (products, softmax exchange,
// barriers) are spread over as many bytes as at head_dim 128
template <int D>
constexpr int tile_keys() { return D == 64 ? 256 : 128; }
constexpr int NROT = 8;                          // rotation warps
constexpr int THREADS = 128 + NROT * 32 + 64;   // softmax + rotation + TMA + MMA
constexpr int WARP_TMA = 4 + NROT;
constexpr int WARP_MMA = 5 + NROT;

constexpr int NKS = 3;    // K ring stages
constexpr int NVS = 3;    // V ring stages
constexpr int HALF_BYTES = 128 * 64 * 2;  // one 64-column SWIZZLE_128B box of a 128-row tile (D = 128)

// Geometry for a head_dim D (64 or 128).  A K or V tile row is D / 64 boxes;
// the Q operand is 16 rows x D.  PV is O^T = V^T P with M = 128: at D = 64 the
// second 64 rows of V^T come from a 2 KB block of zeros (one 16-key k-step),
// so O^T rows 64-127 stay zero and the TMEM layout is that of D = 128.
template <int D>
struct Geo {
  static constexpr int TK = tile_keys<D>();
  static constexpr int NH = D / 64;
  static constexpr int TB = TK * D * 2;             // one K or V tile: 32 KB
  static constexpr int PBOX = 16 * 64 * 2;          // one 64-key box of the P operand
  static constexpr int POPB = PBOX * (TK / 64);     // the P operand: 16 rows x TK keys
  static constexpr int QOPB = 16 * D * 2;
  static constexpr int KSTEPS = D / 16;            // k-steps of S^T = K Q^T
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = NKS * TB;
  static constexpr int OFF_Q = OFF_V + NVS * TB;
  static constexpr int OFF_P = OFF_Q + (QOPB < 1024 ? 1024 : QOPB);
  static constexpr int OFF_Z = OFF_P + 2 * POPB;   // zero block (D = 64)
  // TMEM: S^T of the two tiles in flight, TK / 128 blocks of 16 columns
  // each, then O^T
  static constexpr uint32_t S_COLS = 16 * (TK / 128);
  static constexpr uint32_t COL_O = 2 * S_COLS;
  static constexpr uint32_t TMEM_COLS = COL_O + 16 <= 64 ? 64 : 128;
  static constexpr int SMEM_ALLOC = OFF_Z + (D == 64 ? 2048 : 0) + 1024;
  // rotation warps: CPR 16-byte chunks (8 pairs) per row of the first half,
  // RL row lanes, each thread ROT_ROWS rows of a tile at stride RL
  static constexpr int CPR = D / 16;
  static constexpr int RL = NROT * 32 / CPR;
  static constexpr int ROT_ROWS = TK / RL;
  static constexpr int NENT = 2 * (ROT_ROWS - 1) + 2;  // offset-table entries
};
constexpr int ERR_TIMEOUT = 16;
// kind::f16, D fp32, A/B bf16, M = 128, N = 16; PV reads A (= V^T) MN-major
constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t IDESC_PV = IDESC_QK | (1u << 15);

struct Args {
  const __nv_bfloat16 *q;
  const int32_t *seqlens;
  int Lcap, Hq, Hkv;
  long long w_pre;
  int w0, plain, chunk, nsplit;
  int window;  // sliding-window width (0: none)
  float *part_o, *part_ml;
  int *err;
  // balanced plan (fewer (sequence, kv head) pairs than SMs): one CTA per
  // SM, units sized on the device from the lengths; CTA 0 writes per
  // sequence (first unit, units per kv head) for the combine
  int balanced, batch, max_seqlen;
  int2 *plan_tab;
  // outputs, for the sequences with no key under the balanced plan
  __nv_bfloat16 *out;
  float *lse;
};

constexpr int NSM = 148;

// The balanced plan, computed by one warp of every CTA from the lengths on
// the device (so a captured step replays correctly).  Sequence b attends to
// n_b keys, t_b = ceil(n_b / TK) tiles; a unit is up to k tiles of one
// (sequence, kv head), so (sequence b, kv head) splits into ceil(t_b / k)
// units.  k is the smallest tile count whose units fit one wave (sum over b
// of Hkv * ceil(t_b / k) <= NSM): the longest unit, which sets the step
// time, is then as short as one wave allows.  The warp tests 32 candidate
// k at once and narrows the range until one is left.  Units are numbered
// sequence-major, then kv head, then split.  plan_s receives (b, kv head,
// split, keys per unit, L_b, first key) of this CTA's unit, or b = -1; CTA 0
// writes (first unit, units per kv head) of every sequence to the table (the
// combine's map) and the output of every sequence with no key (zeros, LSE
// -inf).  s_t, s_L, s_jw: NSM ints of shared memory each.  Out of line, so
// that the kernel's loops stay compact.  Requires B * Hkv < NSM (B < NSM).
__device__ __noinline__ void plan_balanced(const Args &p, int TK, int D, int lane, int *plan_s, int *s_t, int *s_L,
                                           int *s_jw) {
  const unsigned full = 0xffffffffu;
  const int B = p.batch;
  int T = 0, nne = 0, tmax = 0;
#pragma unroll 1
  for (int b = lane; b < B; b += 32) {
    int L = p.seqlens[b];
    if (L < 0 || L > p.Lcap || L > p.max_seqlen) L = 0;  // outside the contract: no key
    const int jw = p.window > 0 ? max(0, L - p.window) : 0;
    const int t = (L - jw + TK - 1) / TK;
    s_t[b] = t;
    s_L[b] = L;
    s_jw[b] = jw;
    T += t;
    nne += t > 0 ? 1 : 0;
    tmax = max(tmax, t);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    T += __shfl_xor_sync(full, T, o);
    nne += __shfl_xor_sync(full, nne, o);
    tmax = max(tmax, __shfl_xor_sync(full, tmax, o));
  }
  __syncwarp();
  const int S = NSM / p.Hkv;  // units per kv head in one wave (>= B >= nne)
  int k = 1;
  if (T > 0) {
    // below ceil(T / S) the units exceed S; at hi they fit: either
    // sum(t_b / k + 1) <= S, or k = tmax (one unit per sequence)
    int hi = S > nne ? (T + (S - nne) - 1) / (S - nne) : tmax;
    hi = min(max(hi, 1), tmax);
    int lo = min(max((T + S - 1) / S, 1), hi);
#pragma unroll 1
    while (lo < hi) {
      // candidates nondecreasing over the lanes, the last one hi
      const int step = (hi - lo + 30) / 31;
      const int kc = min(lo + step * lane, hi);
      int units = 0;
#pragma unroll 1
      for (int b = 0; b < B; ++b) units += (s_t[b] + kc - 1) / kc;
      const unsigned fits = __ballot_sync(full, units <= S);  // a suffix of the lanes, lane 31 included
      const int f = __ffs(fits) - 1;
      const int kf = __shfl_sync(full, kc, f);
      const int kp = __shfl_sync(full, kc, f > 0 ? f - 1 : 0);
      lo = min(f > 0 ? kp + 1 : lo, kf);
      hi = kf;
    }
    k = lo;
  }
  // locate this CTA's unit: exclusive prefix of Hkv * ceil(t_b / k) over b
  const int u = blockIdx.x;
  if (lane == 0) plan_s[0] = -1;
  __syncwarp();
  int carry = 0;
#pragma unroll 1
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const int ns = b < B ? (s_t[b] + k - 1) / k : 0;
    int inc = ns * p.Hkv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    const int base = carry + inc - ns * p.Hkv;  // exclusive
    if (b < B) {
      if (u == 0) p.plan_tab[b] = make_int2(base, ns);
      if (ns > 0 && u >= base && u < base + ns * p.Hkv) {
        const int kvh = (u - base) / ns;
        plan_s[0] = b;
        plan_s[1] = kvh;
        plan_s[2] = u - base - kvh * ns;
        plan_s[3] = k * TK;
        plan_s[4] = s_L[b];
        plan_s[5] = s_jw[b];
      }
    }
    carry += __shfl_sync(full, inc, 31);
  }
  if (u == 0) {
    // sequences with no key: no unit writes them
#pragma unroll 1
    for (int b = 0; b < B; ++b) {
      if (s_t[b] == 0) {
        uint4 *o4 = reinterpret_cast<uint4 *>(p.out + (size_t)b * p.Hq * D);
        for (int idx = lane; idx < p.Hq * D / 8; idx += 32) o4[idx] = make_uint4(0u, 0u, 0u, 0u);
        if (p.lse != nullptr)
          for (int h = lane; h < p.Hq; h += 32) p.lse[(size_t)b * p.Hq + h] = -INFINITY;
      }
    }
  }
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
               : "memory");
}
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {  // K-major, SWIZZLE_128B
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {  // MN-major, SWIZZLE_128B
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// packed fp32 pairs: one instruction computes both lanes (sm_100 f32x2)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float2 f) {
  __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 x;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "r"(a));
  return x;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 x) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w)
               : "memory");
}

// byte offset of (row, 16-byte chunk) in a 16-row K-major SWIZZLE_128B operand
// half (rows 128 B apart, chunk XOR-swizzled by row % 8)
__device__ __forceinline__ int op_off(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

template <int GS, int D>
__global__ void __launch_bounds__(THREADS, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                 const __grid_constant__ Args p, const __grid_constant__ InvFreq inv) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_kf[NKS], bar_kr[NKS], bar_ke[NKS], bar_vf[NVS], bar_ve[NVS], bar_sf[2],
      bar_pr[2], bar_q, bar_od, bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ float red[2][4][8];
  // [entry][cos, sin][16-byte slot]: the 8 values of a chunk sit in slots
  // 2 lc and 2 lc + 1, swapped for lc >= 4, so the 8 lanes of a phase (8
  // distinct chunks) read 8 distinct bank groups
  __shared__ float4 otab[Geo<D>::NENT][2][16];

  using GG = Geo<D>;
  constexpr int TK = Geo<D>::TK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's (sequence, kv head, split, keys per split, length, first
  // key): from the grid, or (balanced) from the plan; read back from shared
  // memory by every role
  __shared__ int plan_s[6];
  __shared__ int s_t[NSM], s_L[NSM], s_jw[NSM];
  if (!p.balanced) {
    const int split = blockIdx.x, chunk = p.chunk;
    int L = p.seqlens[blockIdx.z];
    if (L < 0 || L > p.Lcap || L > p.max_seqlen) L = 0;  // outside the contract: no key
    // a sliding-window layer sees keys jw .. L-1 only; the splits cover them
    int jw = p.window > 0 ? max(0, L - p.window) : 0;
    if (L - jw > p.nsplit * chunk) L = jw = 0;  // more keys than the planned splits hold
    if (jw + split * chunk >= L) {
      // no key in this split: an empty partial
      const size_t pidx = ((size_t)blockIdx.z * p.Hq + (size_t)blockIdx.y * GS) * p.nsplit + split;
      for (int idx = threadIdx.x; idx < GS * D; idx += THREADS)
        p.part_o[(pidx + (size_t)(idx / D) * p.nsplit) * D + idx % D] = 0.f;
      if (threadIdx.x < GS) {
        p.part_ml[(pidx + (size_t)threadIdx.x * p.nsplit) * 2 + 0] = -INFINITY;
        p.part_ml[(pidx + (size_t)threadIdx.x * p.nsplit) * 2 + 1] = 0.f;
      }
      return;
    }
    if (threadIdx.x == 0) {
      plan_s[0] = blockIdx.z;
      plan_s[1] = blockIdx.y;
      plan_s[2] = split;
      plan_s[3] = chunk;
      plan_s[4] = L;
      plan_s[5] = jw;
    }
  }

  const uint32_t sbase = (su32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (sbase - su32(smem_raw));

  if (threadIdx.x == 0) {
    for (int s = 0; s < NKS; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_kr[s], NROT * 32);
      mbar_init(&bar_ke[s], 1);
    }
    for (int s = 0; s < NVS; ++s) {
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_sf[s], 1);
      mbar_init(&bar_pr[s], 128);
    }
    mbar_init(&bar_q, 128);
    mbar_init(&bar_od, 1);
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == WARP_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_slot)),
                 "r"(GG::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // the balanced plan runs on a rotation warp beside the set-up above
  if (p.balanced && warp == 4) plan_balanced(p, TK, D, lane, plan_s, s_t, s_L, s_jw);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_slot;
  if (plan_s[0] < 0) {  // balanced plan: no unit for this CTA (uniform)
    if (warp == WARP_MMA)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(GG::TMEM_COLS));
    return;
  }
  const int b = plan_s[0], kvh = plan_s[1], split = plan_s[2], chunk = plan_s[3], L = plan_s[4], jw = plan_s[5];
  const int kb = jw + split * chunk;
  const int ke = min(L, kb + chunk);
  const int n = ke - kb;  // >= 1
  // partial rows of this CTA's heads g: pidx + g * pstride (balanced: the
  // unit's GS rows; otherwise (sequence, head, split) with nsplit splits)
  const size_t pidx = p.balanced ? (size_t)blockIdx.x * GS
                                 : ((size_t)b * p.Hq + (size_t)kvh * GS) * p.nsplit + split;
  const size_t pstride = p.balanced ? 1 : (size_t)p.nsplit;
  const int ntiles = (n + TK - 1) / TK;
  const int row0 = b * p.Lcap + kb;
  const int i = L - 1;
  const int G = p.plain ? 1 : (int)group_size(L, p.w_pre);
  const bool bif = G > 1;
  const int j_local = (int)max(0LL, (long long)L - (long long)p.w0);  // keys >= j_local are local


  if (warp == WARP_TMA) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      int nk = 0, nv = 0;
      bool ok = true;
      for (int u = 0; u < ntiles && ok; ++u) {
        const int sk = u % NKS, sv = u % NVS;
        if (u >= NKS && !(ok = wait_b(&bar_ke[sk], ((u / NKS) - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT))) break;
        mbar_expect_tx(&bar_kf[sk], GG::TB);
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load(&mK, &bar_kf[sk], sbase + GG::OFF_K + sk * GG::TB + hf * HALF_BYTES, 64 * hf, kvh, row0 + u * TK);
        ++nk;
        if (u >= NVS && !(ok = wait_b(&bar_ve[sv], ((u / NVS) - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT))) break;
        mbar_expect_tx(&bar_vf[sv], GG::TB);
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load(&mV, &bar_vf[sv], sbase + GG::OFF_V + sv * GG::TB + hf * HALF_BYTES, 64 * hf, kvh, row0 + u * TK);
        ++nv;
      }
      for (int u = max(0, nk - NKS); u < nk; ++u) wait_drain(&bar_kf[u % NKS], (u / NKS) & 1, p.err, ERR_TIMEOUT);
      for (int u = max(0, nv - NVS); u < nv; ++u) wait_drain(&bar_vf[u % NVS], (u / NVS) & 1, p.err, ERR_TIMEOUT);
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer =======================
    // A small scheduler: QK of tile uq as soon as its rotated K is ready (and
    // its S buffer is free, i.e. PV of tile uq-2 issued), PV of tile up as
    // soon as its P and V are ready.  Neither waits on the other's inputs.
    if (lane == 0) {
      bool ok = wait_b(&bar_q, 0, &abort_flag, p.err, ERR_TIMEOUT);
      int uq = 0, up = 0;
      uint64_t t_idle = gtime();
      uint32_t spins = 0;
      while (ok && up < ntiles) {
        bool progressed = false;
        if (uq < ntiles && uq - up < 2 && mbar_test(&bar_kr[uq % NKS], (uq / NKS) & 1)) {
          fence_after();
          const int sk = uq % NKS;
          const uint32_t ka = sbase + GG::OFF_K + sk * GG::TB;
          const uint32_t qa = sbase + GG::OFF_Q;
#pragma unroll
          for (int mb = 0; mb < TK / 128; ++mb) {  // keys 128 mb .. 128 mb + 127 (rows 128 B apart at D = 64)
#pragma unroll
            for (int kk = 0; kk < GG::KSTEPS; ++kk) {
              const uint32_t ko = mb * 128 * 128 + (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
              const uint32_t qo = (kk >> 2) * (GG::QOPB / 2) + (kk & 3) * 32;
              mma_ss(tmem + (uint32_t)((uq & 1) * GG::S_COLS + 16 * mb), desc_k(ka + ko), desc_k(qa + qo), IDESC_QK,
                     kk > 0 ? 1u : 0u);
            }
          }
          commit(&bar_sf[uq & 1]);
          commit(&bar_ke[sk]);
          ++uq;
          progressed = true;
        }
        if (up < uq && mbar_test(&bar_pr[up & 1], (up >> 1) & 1) &&
            mbar_test(&bar_vf[up % NVS], (up / NVS) & 1)) {
          fence_after();
          const int sv = up % NVS;
          const uint32_t va = sbase + GG::OFF_V + sv * GG::TB;
          const uint32_t pa = sbase + GG::OFF_P + (up & 1) * GG::POPB;
#pragma unroll
          for (int kk = 0; kk < TK / 16; ++kk) {
            // the second 64 rows of V^T: the tile's second box, or (D = 64)
            // the zero block, which lies after every V stage
            const uint32_t vk = va + kk * 2048;
            const uint32_t lbo = D == 128 ? (uint32_t)HALF_BYTES : sbase + (uint32_t)GG::OFF_Z - vk;
            mma_ss(tmem + GG::COL_O, desc_mn(vk, lbo), desc_k(pa + (kk >> 2) * GG::PBOX + (kk & 3) * 32), IDESC_PV,
                   (up > 0 || kk > 0) ? 1u : 0u);
          }
          commit(&bar_ve[sv]);
          commit(&bar_od);
          ++up;
          progressed = true;
        }
        if (progressed) {
          spins = 0;
          t_idle = gtime();
        } else if ((++spins & 31u) == 0) {
          if (abort_flag) ok = false;
          else if (gtime() - t_idle > *(volatile unsigned long long *)&g_wait_limit_ns) {
            abort_flag = 1;
            atomicOr(p.err, ERR_TIMEOUT);
            ok = false;
          }
        }
      }
      commit(&bar_drain);
      wait_drain(&bar_drain, 0, p.err, ERR_TIMEOUT);
    }
  } else if (warp >= 4) {
    // ======================= rotation warps =======================
    // Thread t owns one 16-byte chunk (8 pairs) of the first half of rows
    // r0 + RL m of every tile, together with the partner chunk of the second
    // half (elements k + D/2).  Its row-r0 rotation (the tile base) advances
    // once per tile; the other rows compose the base with a fixed offset
    // rotation, so the rows of a tile do not wait on one another.  With
    // J = j0 + r0 and rho = J mod G, the offset of row m is
    //   n(J + RL m) - n(J) = RL m - floor(RL m / G) - [rho + (RL m mod G) >= G]
    // and the base advances by TK - floor(TK / G) - [rho + (TK mod G) >= G]:
    // each a choice between two increments, tabulated once per CTA.
    constexpr int RS = GG::RL;        // row stride of one thread
    constexpr int NR = GG::ROT_ROWS;  // rows of one thread per tile
    constexpr int EB = GG::NENT - 2;  // first base-advance entry
    const int t = threadIdx.x - 128;
    int r0, lc;                       // first row; logical chunk (pairs 8 lc ..)
    if constexpr (D == 128) {
      r0 = t >> 3;
      lc = (t & 7) ^ (r0 & 7);        // 8 lanes of a phase: 8 chunks of one row
    } else {
      // 8 lanes of a phase: rows a and a + 4 (their swizzles differ by 4, so
      // the 4 + 4 chunks they touch fall in distinct bank groups)
      const int ph = t >> 3;
      r0 = ((ph >> 2) << 3) + (ph & 3) + 4 * ((t >> 2) & 1);
      lc = t & 3;
    }
    // byte offsets in a tile row of this thread's two chunks (rows r0 + RS m
    // share r0's swizzle: RS is a multiple of 8)
    const int offa = D == 128 ? ((lc ^ (r0 & 7)) << 4) : ((lc ^ (r0 & 7)) << 4);
    const int offb = D == 128 ? HALF_BYTES + ((lc ^ (r0 & 7)) << 4) : (((lc + 4) ^ (r0 & 7)) << 4);
    float bc[8], bs[8];               // rotation of row r0 of the current tile
    int rho = 0, sb = 0;
    int smm[NR];
#pragma unroll
    for (int m = 0; m < NR; ++m) smm[m] = 0;
    if (bif) {
      if (t < GG::NENT * GG::CPR) {
        // offset table: entries 2(m-1) + carry for rows m = 1..NR-1, EB + carry
        // for the base advance
        const int tl = t % GG::CPR, en = t / GG::CPR;
        const int span = en < EB ? RS * (en / 2 + 1) : TK;
        const int d = span - span / G - (en & 1);
        float c[8], sn[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) angle_cs(d, inv.v[tl * 8 + e], c[e], sn[e]);
        const int sw = (tl >> 2) & 1;
        otab[en][0][2 * tl + sw] = make_float4(c[0], c[1], c[2], c[3]);
        otab[en][0][2 * tl + (sw ^ 1)] = make_float4(c[4], c[5], c[6], c[7]);
        otab[en][1][2 * tl + sw] = make_float4(sn[0], sn[1], sn[2], sn[3]);
        otab[en][1][2 * tl + (sw ^ 1)] = make_float4(sn[4], sn[5], sn[6], sn[7]);
      }
      const int jf = kb + r0;
      const int ni = corr_n(i, G);
#pragma unroll
      for (int e = 0; e < 8; ++e) angle_cs(corr_n(jf, G) - ni, inv.v[lc * 8 + e], bc[e], bs[e]);
      rho = jf % G;
#pragma unroll
      for (int m = 1; m < NR; ++m) smm[m] = (RS * m) % G;
      sb = TK % G;
      asm volatile("bar.sync 2, %0;" ::"n"(NROT * 32) : "memory");
    }
    // (c, s) <- (c, s) x offset entry en of this thread's chunk
    auto compose = [&](int en, float (&c)[8], float (&sn)[8]) {
      const int sw = (lc >> 2) & 1;
      const float4 c0 = otab[en][0][2 * lc + sw], c1 = otab[en][0][2 * lc + (sw ^ 1)];
      const float4 s0 = otab[en][1][2 * lc + sw], s1 = otab[en][1][2 * lc + (sw ^ 1)];
      const float2 oc[4] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w), make_float2(c1.x, c1.y),
                            make_float2(c1.z, c1.w)};
      const float2 os[4] = {make_float2(s0.x, s0.y), make_float2(s0.z, s0.w), make_float2(s1.x, s1.y),
                            make_float2(s1.z, s1.w)};
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        const float2 b_c = make_float2(bc[2 * e2], bc[2 * e2 + 1]);
        const float2 b_s = make_float2(bs[2 * e2], bs[2 * e2 + 1]);
        const float2 cc = sub2(mul2(b_c, oc[e2]), mul2(b_s, os[e2]));
        const float2 ss = fma2(b_s, oc[e2], mul2(b_c, os[e2]));
        c[2 * e2] = cc.x;
        c[2 * e2 + 1] = cc.y;
        sn[2 * e2] = ss.x;
        sn[2 * e2 + 1] = ss.y;
      }
    };
    auto advance_base = [&]() {
      const int cy = rho + sb >= G ? 1 : 0;
      float c[8], sn[8];
      compose(EB + cy, c, sn);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        bc[e] = c[e];
        bs[e] = sn[e];
      }
      rho += sb - cy * G;
    };
    bool ok = true;
    for (int u = 0; u < ntiles && ok; ++u) {
      const int sk = u % NKS;
      const int j0 = kb + u * TK;
      const bool rot_tile = bif && j0 < j_local;
      ok = __all_sync(0xffffffffu, wait_b(&bar_kf[sk], (u / NKS) & 1, &abort_flag, p.err, ERR_TIMEOUT));
      if (!ok) break;
      if (rot_tile) {
        const uint32_t kt = sbase + GG::OFF_K + sk * GG::TB;
        // every row's data is read before any row is written back, so the
        // shared-memory latencies overlap
        uint4 xa[NR], xb[NR];
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          const int r = r0 + RS * m;
          xa[m] = lds128(kt + r * 128 + offa);
          xb[m] = lds128(kt + r * 128 + offb);
        }
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          const int r = r0 + RS * m;
          if (j0 + r < j_local) {
            float rc[8], rs[8];
            if (m == 0) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                rc[e] = bc[e];
                rs[e] = bs[e];
              }
            } else {
              compose(2 * (m - 1) + (rho + smm[m] >= G ? 1 : 0), rc, rs);
            }
            uint32_t *ua = reinterpret_cast<uint32_t *>(&xa[m]), *ub = reinterpret_cast<uint32_t *>(&xb[m]);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              const float2 fa = bf2_to_f2(ua[e2]), fb = bf2_to_f2(ub[e2]);
              const float2 cc = make_float2(rc[2 * e2], rc[2 * e2 + 1]);
              const float2 ss = make_float2(rs[2 * e2], rs[2 * e2 + 1]);
              ua[e2] = f2_to_bf2(fma2(fa, cc, mul2(fb, ss)));
              ub[e2] = f2_to_bf2(sub2(mul2(fb, cc), mul2(fa, ss)));
            }
            sts128(kt + r * 128 + offa, xa[m]);
            sts128(kt + r * 128 + offb, xb[m]);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        advance_base();
      } else if (bif) {
        // no remote key in this tile: only advance the base
        advance_base();
      }
      mbar_arrive(&bar_kr[sk]);
    }
  } else {
    // ======================= softmax warpgroup =======================
    const int r = threadIdx.x;  // key row of the tile (and r + 128 ..) / head-dim row of O^T / TMEM lane
    constexpr int KPT = TK / 128;  // keys of a tile per thread
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
    // Q operand: rows h < GS hold the query heads, rows GS..15 zero; also zero
    // the padding rows of both P buffers, and (D = 64) the zero block
    {
      const int h = r >> 3, c = r & 7;
#pragma unroll
      for (int hf = 0; hf < GG::NH; ++hf) {
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (h < GS)
          val = *reinterpret_cast<const uint4 *>(p.q + ((size_t)b * p.Hq + (size_t)kvh * GS + h) * D + hf * 64 +
                                                 c * 8);
        *reinterpret_cast<uint4 *>(gbase + GG::OFF_Q + hf * (GG::QOPB / GG::NH) + op_off(h, c)) = val;
      }
      if (h >= GS)
#pragma unroll
        for (int hf = 0; hf < TK / 64; ++hf)
#pragma unroll
          for (int pb = 0; pb < 2; ++pb)
            *reinterpret_cast<uint4 *>(gbase + GG::OFF_P + pb * GG::POPB + hf * GG::PBOX + op_off(h, c)) =
                make_uint4(0u, 0u, 0u, 0u);
      if constexpr (D == 64) reinterpret_cast<uint4 *>(gbase + GG::OFF_Z)[r] = make_uint4(0u, 0u, 0u, 0u);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bar_q);
    }
    float m_run[GS], l_part[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      m_run[g] = -INFINITY;
      l_part[g] = 0.f;
    }
    bool ok = true;
    int u = 0;
    for (; u < ntiles && ok; ++u) {
      const int bsel = u & 1;
      // on a timeout this warp carries on with garbage until the barrier below,
      // where every warp of the group sees the abort and leaves together
      wait_b(&bar_sf[bsel], (u >> 1) & 1, &abort_flag, p.err, ERR_TIMEOUT);
      fence_after();
      // keys r + 128 mb of the tile
      float s[KPT][GS];
      bool valid[KPT];
#pragma unroll
      for (int mb = 0; mb < KPT; ++mb) {
        uint32_t sr[8];
        tmem_ld8(tmem + lane_base + (uint32_t)(bsel * GG::S_COLS + 16 * mb), sr);
        valid[mb] = kb + u * TK + 128 * mb + r < ke;
#pragma unroll
        for (int g = 0; g < GS; ++g) s[mb][g] = valid[mb] ? __uint_as_float(sr[g]) * sl2 : -INFINITY;
      }
      // block-wide tile max per head
      float mt[GS];
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        float x = s[0][g];
#pragma unroll
        for (int mb = 1; mb < KPT; ++mb) x = fmaxf(x, s[mb][g]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
        mt[g] = x;
      }
      // exchange the four warps' maxima through shared memory; the named
      // barrier also ORs the abort state so that all four warps leave the
      // loop at the same tile (keeping their barrier counts equal)
      if (lane == 0)
#pragma unroll
        for (int g = 0; g < GS; ++g) red[bsel][warp][g] = mt[g];
      if (bar_red_or(1, 128, abort_flag != 0)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int g = 0; g < GS; ++g)
        mt[g] = fmaxf(fmaxf(red[bsel][0][g], red[bsel][1][g]), fmaxf(red[bsel][2][g], red[bsel][3][g]));
      // lazy rescale: only when a head's max grows by more than 2^8
      float f[GS];
      bool any = false;
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        const float mn = fmaxf(m_run[g], mt[g]);
        f[g] = 1.f;
        if (m_run[g] == -INFINITY) {
          m_run[g] = mn;
        } else if (mn > m_run[g] + 8.f) {
          f[g] = exp2f(m_run[g] - mn);
          m_run[g] = mn;
          any = true;
        }
      }
      if (any) {  // uniform over the warpgroup (all threads see the same maxima)
        // O holds PV of tiles < u once PV_{u-1} is complete
        wait_b(&bar_od, (u - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT);
        fence_after();
        uint32_t orow[8];
        tmem_ld8(tmem + lane_base + GG::COL_O, orow);
#pragma unroll
        for (int g = 0; g < GS; ++g) orow[g] = __float_as_uint(__uint_as_float(orow[g]) * f[g]);
        tmem_st8(tmem + lane_base + GG::COL_O, orow);
#pragma unroll
        for (int g = 0; g < GS; ++g) l_part[g] *= f[g];
      }
      // P (bf16) into the B operand of the PV MMA: row g = head, column r = key
#pragma unroll
      for (int mb = 0; mb < KPT; ++mb) {
        const int kr = r + 128 * mb;  // key row of the tile: 64-key box kr / 64
        uint8_t *pbuf = gbase + GG::OFF_P + bsel * GG::POPB + (kr >> 6) * GG::PBOX;
        const int chunk = (kr & 63) >> 3;
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          const float pr = valid[mb] ? ex2(s[mb][g] - m_run[g]) : 0.f;
          l_part[g] += pr;
          *reinterpret_cast<__nv_bfloat16 *>(pbuf + op_off(g, chunk) + (kr & 7) * 2) = __float2bfloat16_rn(pr);
        }
      }
      // a partial last tile: zero the V rows past the last key (the cache may
      // hold anything there, and 0 * NaN would poison the PV product)
      if (u == ntiles - 1 && (n % TK) != 0) {
        const int sv = u % NVS;
        wait_b(&bar_vf[sv], (u / NVS) & 1, &abort_flag, p.err, ERR_TIMEOUT);
        if (!abort_flag) {
          uint8_t *vt = gbase + GG::OFF_V + sv * GG::TB;
#pragma unroll
          for (int mb = 0; mb < KPT; ++mb)
            if (!valid[mb])
#pragma unroll
              for (int hf = 0; hf < GG::NH; ++hf)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  *reinterpret_cast<uint4 *>(vt + hf * HALF_BYTES + (r + 128 * mb) * 128 + c * 16) =
                      make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // last tile: PV of the previous tile must be complete before this
      // tile's PV is released, so exactly one PV is outstanding at the end
      if (u == ntiles - 1 && u > 0) wait_b(&bar_od, (u - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      fence_before();
      mbar_arrive(&bar_pr[bsel]);
    }
    // ---- epilogue: this split's partial (m, l, O) per head
    if (ok && u > 0) wait_b(&bar_od, (u - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT);
    float lsum[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      float x = l_part[g];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      lsum[g] = x;
    }
    __shared__ float lred[4][8];
    if (lane == 0)
#pragma unroll
      for (int g = 0; g < GS; ++g) lred[warp][g] = lsum[g];
    if (bar_red_or(1, 128, abort_flag != 0)) ok = false;
    if (ok) {
      fence_after();
      uint32_t orow[8];
      tmem_ld8(tmem + lane_base + GG::COL_O, orow);
      if (r < D)  // O^T row r is head_dim element r
#pragma unroll
        for (int g = 0; g < GS; ++g) p.part_o[(pidx + (size_t)g * pstride) * D + r] = __uint_as_float(orow[g]);
      if (r < GS) {
        const float l = lred[0][r] + lred[1][r] + lred[2][r] + lred[3][r];
        p.part_ml[(pidx + (size_t)r * pstride) * 2 + 0] = m_run[r];
        p.part_ml[(pidx + (size_t)r * pstride) * 2 + 1] = l;
      }
    } else {
      if (r < D)
        for (int g = 0; g < GS; ++g) p.part_o[(pidx + (size_t)g * pstride) * D + r] = 0.f;
      if (r < GS) {
        p.part_ml[(pidx + (size_t)r * pstride) * 2 + 0] = -INFINITY;
        p.part_ml[(pidx + (size_t)r * pstride) * 2 + 1] = 0.f;
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(GG::TMEM_COLS));
  }
}

}  // namespace dtc

// ------------------------------------------------------------------ host
// Split plan: one CTA per SM (the rings take ~200 KB of shared memory), one
// wave of 148, whole tiles (128 keys at head_dim 128, 256 at 64).
void decode_tc_plan(int batch, int Hkv, int D, int max_seqlen, int *nsplit, int *chunk) {
  const long long bh = (long long)batch * (long long)Hkv;
  const int ns0 = bh >= 148 ? 1 : (int)(148 / max(1LL, bh));
  const int maxL = max(1, max_seqlen);
  int c = (maxL + ns0 - 1) / ns0;
  const int tk = D == 64 ? dtc::tile_keys<64>() : dtc::tile_keys<128>();
  c = (c + tk - 1) / tk * tk;
  *chunk = c;
  *nsplit = (maxL + c - 1) / c;
}

cudaError_t launch_decode_tc(int GS, int D, const CUtensorMap &mK, const CUtensorMap &mV, const __nv_bfloat16 *q,
                             const int32_t *seqlens, int B, int Lcap, int max_seqlen, int Hq, int Hkv,
                             long long w_pre, int w0, int window, const InvFreq &inv, int plain, int nsplit,
                             int chunk, float *part_o, float *part_ml, int2 *plan_tab, __nv_bfloat16 *out,
                             float *lse, int *err, cudaStream_t st) {
  dtc::Args a;
  a.q = q;
  a.seqlens = seqlens;
  a.Lcap = Lcap;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.w_pre = w_pre;
  a.w0 = w0;
  a.plain = plain;
  a.window = window;
  a.chunk = chunk;
  a.nsplit = nsplit;
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.err = err;
  // balanced: one CTA per SM, units planned on the device
  a.balanced = plan_tab != nullptr;
  a.batch = B;
  a.max_seqlen = max_seqlen;
  a.plan_tab = plan_tab;
  a.out = out;
  a.lse = lse;
  const dim3 grid = a.balanced ? dim3(dtc::NSM, 1, 1) : dim3(nsplit, Hkv, B);
  cudaError_t e;
#define JL_DTC(GG, DD)                                                                                    \
  e = cudaFuncSetAttribute(dtc::decode_tc_kernel<GG, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,       \
                           dtc::Geo<DD>::SMEM_ALLOC);                                                        \
  if (e != cudaSuccess) return e;                                                                          \
  dtc::decode_tc_kernel<GG, DD><<<grid, dtc::THREADS, dtc::Geo<DD>::SMEM_ALLOC, st>>>(mK, mV, a, inv);
  if (D == 128) {
    switch (GS) {
      case 1: JL_DTC(1, 128) break;
      case 2: JL_DTC(2, 128) break;
      case 4: JL_DTC(4, 128) break;
      case 8: JL_DTC(8, 128) break;
      default: return cudaErrorInvalidValue;
    }
  } else if (D == 64) {
    switch (GS) {
      case 1: JL_DTC(1, 64) break;
      case 2: JL_DTC(2, 64) break;
      case 4: JL_DTC(4, 64) break;
      case 8: JL_DTC(8, 64) break;
      default: return cudaErrorInvalidValue;
    }
  } else {
    return cudaErrorInvalidValue;
  }
#undef JL_DTC
  return cudaGetLastError();
}

}  // namespace jl

namespace jl {
// Test hook: the limit of the bounded waits of this file's kernels.
cudaError_t set_wait_limit_decode_tc(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}
}  // namespace jl
