// Tensor-core prefill kernels for Dynamic Bifocal RoPE attention (sm_100a).
//
// Jet-Long technical summary, §2 "Mecanismos de Eficiência de Inferência":
// the local window (base RoPE), the full causal pass over grouped queries and
// keys, and the window pass over grouped queries and keys are merged by
// inclusion–exclusion with LSE statistics, which gives the exact
// distance-routed attention (§1 "Janela Local" / "Janela Remota").  These
// kernels compute that exact value in one causal pass: every (query tile,
// key tile) pair is visited with the base operands where all its distances
// are < w0, with the grouped operands where all are >= w0, and twice (once
// each, complementary masks) on the tile that straddles d = w0; one online
// softmax runs over all visits.
//
// The grouped operands come from the on-the-fly correction rotation of §2
// "Rotação de Correção On-the-Fly", applied in the kernels and never written
// back: the query tile is rotated once per CTA by R(f(i) - i), and each key
// tile of a grouped visit is rotated in place in shared memory by
// R(f(j) - j), between its TMA load and its QK products, by a warpgroup of
// its own (KeyCorrection below).
//
// Two kernels, both templated on the head_dim D (64 or 128), both organised
// in whole warpgroups so that `setmaxnreg` can move registers from the
// producer, MMA and rotation roles to the softmax warpgroups:
//   bifocal_prefill2_kernel  two query heads of one GQA group per CTA (even
//                            groups), 4 warpgroups; layout above its definition
//   bifocal_prefill_kernel   one query head per CTA (odd groups), 3 warpgroups
//
// Every mbarrier wait is bounded (%globaltimer); on expiry the kernel records
// an error code, tells the other roles to stop, waits (bounded) for its own
// copies and MMAs in flight, frees TMEM and returns.
#include <cuda.h>

#include <type_traits>

#include "../../include/jetlong.h"
#include "jl_common.cuh"
#define JL_WAITS_INLINE 1  // these kernels use setmaxnreg: no calls
#include "jl_ptx.cuh"

namespace jl {
namespace tc {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int P1_NKS = 3;  // K ring stages (one head per CTA)
constexpr int NVS = 2;   // V ring stages (one head per CTA)
constexpr int HALF_BYTES = BM * 64 * 2;  // one 64-column SWIZZLE_128B box of a 128-row tile
constexpr int OFF_Q = 0;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 256;
constexpr int HI_INF = 1 << 30;

// one head per CTA: warpgroups softmax | producers + MMA | key correction
constexpr int P1_THREADS = 384;
constexpr uint32_t P1_REG_SOFTMAX = 232, P1_REG_IO = 104, P1_REG_KCORR = 168;  // 232 + 104 + 168 = 3 x 168
// two heads per CTA: softmax A | softmax B | key correction | producers + MMA
constexpr int P2_THREADS = 512;
constexpr uint32_t P2_REG_SOFTMAX = 176, P2_REG_KCORR = 96, P2_REG_IO = 64;  // 2 x 176 + 96 + 64 = 4 x 128

// error codes (bit flags) written to the workspace error word
constexpr int ERR_TIMEOUT_PRODUCER = 1;
constexpr int ERR_TIMEOUT_MMA = 2;
constexpr int ERR_TIMEOUT_SOFTMAX = 4;
constexpr int ERR_TIMEOUT_KCORR = 32;

struct Params {
  const int32_t *cu;    // query prefix sums [batch + 1]
  const int32_t *cu_k;  // key prefix sums [batch + 1]
  int batch, T, Hq, Hkv;
  int Tk;               // key tokens
  long long w_pre;
  int w0, plain;
  int window;           // sliding-window width (0: none)
  int kg_pre;           // 1: grouped keys were written by prerotate_k_kernel (ablation)
  __nv_bfloat16 *out;
  float *lse;
  int *err;
  float sl2;  // log2(e) / sqrt(D)
};

template <uint32_t R>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R) : "memory");
}
template <uint32_t R>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   su32(bar))
               : "memory");
}
// tcgen05.mma, kind::f16, D in TMEM: A and B from shared memory (ss) or A
// from TMEM (ts).  The shared-memory descriptors come as 32-bit halves: the
// low half (start address) varies by stage and k-step, the high half is
// fixed, so the single issuing thread spends one add per operand per k-step.
__device__ __forceinline__ void umma_ss_lh(uint32_t d, uint32_t alo, uint32_t ahi, uint32_t blo, uint32_t bhi,
                                           uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d),
      "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc));
}
template <uint32_t ACC>
__device__ __forceinline__ void umma_ss_lhc(uint32_t d, uint32_t alo, uint32_t ahi, uint32_t blo, uint32_t bhi,
                                            uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d),
      "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "n"(ACC));
}
template <uint32_t ACC>
__device__ __forceinline__ void umma_ts_lhc(uint32_t d, uint32_t a_tmem, uint32_t blo, uint32_t bhi, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "n"(ACC));
}
__device__ __forceinline__ void umma_ts_lh(uint32_t d, uint32_t a_tmem, uint32_t blo, uint32_t bhi, uint32_t idesc,
                                           uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc));
}

#define JL_R32(a) \
  "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), \
  "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]),       \
  "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]),     \
  "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]),     \
  "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
#define JL_W32(a) \
  "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), "r"(a[8]), \
  "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]), "r"(a[16]),    \
  "r"(a[17]), "r"(a[18]), "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]), "r"(a[24]),   \
  "r"(a[25]), "r"(a[26]), "r"(a[27]), "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : JL_R32(r)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31, %32};" ::"r"(taddr),
      JL_W32(r)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// wait::ld that also "redefines" the loaded registers, so no use of them can be
// scheduled before the wait
#define JL_RW32(a) \
  "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]), \
  "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]),       \
  "+r"(a[15]), "+r"(a[16]), "+r"(a[17]), "+r"(a[18]), "+r"(a[19]), "+r"(a[20]), "+r"(a[21]),     \
  "+r"(a[22]), "+r"(a[23]), "+r"(a[24]), "+r"(a[25]), "+r"(a[26]), "+r"(a[27]), "+r"(a[28]),     \
  "+r"(a[29]), "+r"(a[30]), "+r"(a[31])
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : JL_RW32(r) : : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

constexpr int P2_NKS = 3;
constexpr int P2_NVS = 2;
constexpr int P2_OFF_Q = 0;  // Q_A, Q_B

// Tile geometry for a head_dim D (64 or 128): a tile row of D bf16 is D / 64
// SWIZZLE_128B boxes of 64 columns (HALF_BYTES each for 128 rows).  O_x sits
// at TMEM columns COL_O + x * D.
template <int D>
struct Geo {
  static constexpr int NH = D / 64;          // 64-column boxes per tile row
  static constexpr int TB = BM * D * 2;      // one Q, K or V tile
  static constexpr int KSTEPS = D / 16;      // k-steps of a QK product
  // two heads per CTA: Q_A, Q_B, the K ring, the V ring
  static constexpr int OFF_K = P2_OFF_Q + 2 * TB;
  static constexpr int OFF_V = OFF_K + P2_NKS * TB;
  static constexpr int SMEM_ALLOC = OFF_V + P2_NVS * TB + 1024;
  // one head per CTA: Q, Q_g, the K ring, the V ring
  static constexpr int P1_OFF_QG = TB;
  static constexpr int P1_OFF_K = 2 * TB;
  static constexpr int P1_OFF_V = P1_OFF_K + P1_NKS * TB;
  static constexpr int P1_SMEM_ALLOC = P1_OFF_V + NVS * TB + 1024;
  // kind::f16, D fp32, A/B bf16, M = 128, N = D, B (= V) MN-major
  static constexpr uint32_t IDESC_PV =
      (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(D >> 3) << 17) | ((128u >> 4) << 24);
};

// Shared-memory matrix descriptors (tcgen05 format, version 1).
// K-major, 128-byte swizzle: 8-row atoms of 128 B, atoms 1024 B apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// MN-major, 128-byte swizzle: 64 contiguous N elements per 128 B row, 8 K rows
// per 1024 B atom (SBO), N blocks of 64 `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor, kind::f16: D fp32, A/B bf16, M = 128, N = 128.
constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t IDESC_PV = IDESC_QK | (1u << 16);  // B (= V) is MN-major

// --------------------------------------------------------- tile schedule
// A query tile: rows i0..i1 of a sequence with L queries at positions
// off + i (off = Lk - L) over keys 0..Lk-1; G follows Lk.  W > 0 hides keys
// at distance >= W (a sliding-window layer).
struct Tile {
  int L, G, i0, i1, qt, bif, Lk, off, W;
};

// Visits of a query tile, in order: the base visits (pairs with distance
// < min(w0, W)) on key tiles ks_begin .. the last key tile, then the grouped
// visits (key tiles whose pairs include a distance in [w0, W)) on key tiles
// g_begin .. g_begin + n_grp - 1, ascending.  A visit's
// columns c with (p_i - j0 - c) outside [lo, hi] are masked when `mask` is
// set.  Everything is computed from integers in registers (no per-visit
// arrays).
struct Visit {
  int grp, mask, lo, hi;
};

struct VisitPlan {
  int n_grp, n_all, ks_begin, g_begin;
};

__host__ __device__ __forceinline__ VisitPlan make_plan(const Tile &t, int w0) {
  VisitPlan pl;
  const int pmin = t.off + t.i0, pmax = t.off + t.i1;  // row positions
  const int kt_last = pmax / BN;                        // last key tile with a visible key
  // first key tile with a key inside the first row's window: dmin(kt) =
  // pmin - (kt*BN + BN-1) <= W - 1
  const int xw = pmin - t.W + 1;
  const int kt_first = (t.W > 0 && xw > 0) ? xw / BN : 0;
  pl.g_begin = kt_first;
  if (!t.bif) {
    pl.n_grp = 0;
    pl.ks_begin = kt_first;
    pl.n_all = kt_last - kt_first + 1;
    return pl;
  }
  // grouped: dmax(kt) = pmax - kt*BN >= w0, and some grouped distance is
  // inside the window
  const bool any_grp = pmax >= w0 && (t.W == 0 || t.W > w0);
  pl.n_grp = any_grp ? max(0, min(kt_last, (pmax - w0) / BN) - kt_first + 1) : 0;
  // base: dmin(kt) = pmin - (kt*BN + BN-1) <= bl - 1 with bl = min(w0, W);
  // the last key tile always qualifies when bl >= 1
  const int bl = t.W > 0 ? min(w0, t.W) : w0;
  int nstd = 0;
  pl.ks_begin = kt_last + 1;
  if (bl > 0) {
    const int x = pmin - (BN - 1) - (bl - 1);  // need kt*BN >= x
    pl.ks_begin = max(kt_first, x <= 0 ? 0 : min(kt_last, (x + BN - 1) / BN));
    nstd = kt_last - pl.ks_begin + 1;
  }
  pl.n_all = pl.n_grp + nstd;
  return pl;
}

__host__ __device__ __forceinline__ void visit_at(const Tile &t, const VisitPlan &pl, int w0, int v, int &kt,
                                                  Visit &out) {
  const int n_base = pl.n_all - pl.n_grp;
  const bool grp = v >= n_base;
  kt = grp ? pl.g_begin + (v - n_base) : pl.ks_begin + v;
  const int j0 = kt * BN;
  const int j1 = min(j0 + BN - 1, t.Lk - 1);
  const int dmin = t.off + t.i0 - j1, dmax = t.off + t.i1 - j0;
  // the tile holds a key past some row's position (this includes keys at or
  // past Lk: zero-filled, or the next sequence's): the causal mask is needed
  const int causal = j0 + BN - 1 > t.off + t.i0;
  const int whi = t.W > 0 ? t.W - 1 : HI_INF;  // largest visible distance
  if (grp) {
    out = Visit{1, causal || dmin < w0 || dmax > whi, w0, whi};
  } else if (!t.bif) {
    out = Visit{0, causal || dmax > whi, 0, whi};
  } else {
    const int hi = min(w0 - 1, whi);
    out = Visit{0, causal || dmax > hi, 0, hi};
  }
}

// ------------------------------------------------------------ key correction
// §2 "Rotação de Correção On-the-Fly": the grouped branch scores a remote key
// at its grouped position, K_g = R(f(j) - j) K~ = R(-n(j)) K~ with
// n(j) = j - floor(j / G), while the stored keys stay as they are.  One
// warpgroup of the prefill CTA applies that rotation in place to the K tile
// of every grouped visit, in shared memory, after the tile's TMA load and
// before its QK products read it.
//
// Thread t (0..127) owns the 8 pairs k = 8 lc .. 8 lc + 7 (pair k: elements k
// and k + D/2) of RPT consecutive rows r0 .. r0 + RPT - 1 of every tile:
//   D = 128: lc = t % 8, rows 8 (t / 8) ..; element k in box 0 and k + 64 in
//            the same 16-byte chunk of box 1;
//   D = 64:  lc = t % 4, rows 4 (t / 4) ..; chunk lc pairs with chunk lc + 4
//            of the same 128-byte row.
// The eight lanes of each shared-memory phase touch eight distinct 16-byte
// bank groups in both layouts.  From one key to the next, n grows by one
// except where the next key index is a multiple of G, so along its rows a
// thread steps its rotation by R(1) or keeps it.  The rotation of its first
// row advances once per tile by R(delta), delta = n(j + BN) - n(j): with
// BN = b G + sigma and rho = j mod G, delta = BN - b - [rho + sigma >= G], so
// the step is R(BN - b), tabulated per CTA, times R(-1) when the carry is
// set.  Angles are seeded in fp64 (the fp64 sine and cosine of the exact
// integer multiple) and carried in fp32; a CTA advances at most L / BN tile
// steps.
struct KCorrTable {
  float4 v[4][8];  // R(BN - b) per chunk lc: [cos 0-3, cos 4-7, sin 0-3, sin 4-7][lc]
};

__device__ __forceinline__ float2 bf2_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_bf2(float2 f) {
  __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }
// (c, s) <- (c, s) x (c1, s1): rotation angles add
__device__ __forceinline__ void compose2(float2 &c, float2 &s, float2 c1, float2 s1) {
  const float2 cn = __ffma2_rn(c, c1, __fmul2_rn(neg2(s), s1));
  const float2 sn = __ffma2_rn(s, c1, __fmul2_rn(c, s1));
  c = cn;
  s = sn;
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

template <int D, int NSTAGE>
struct KeyCorrection {
  static constexpr int CPR = D / 16;          // 8-pair chunks per row
  static constexpr int RPT = BN * CPR / 128;  // rows per thread per tile
  int lc, r0, G, sigma, rho;
  float2 bc[4], bs[4];  // rotation by n of the thread's first row, pairs (2w, 2w + 1) packed
  float2 c1[4], s1[4];  // R(1)

  // Set-up once per CTA, by all 128 threads of the warpgroup: R(BN - b) into
  // `tab` (then a named barrier over the warpgroup), R(1) and the first
  // tile's rotation in registers.  j_first: the first key of the first
  // grouped visit.
  __device__ __forceinline__ void init(int t, int j_first, int G_, const InvFreq &inv, KCorrTable &tab,
                                       int bar_id) {
    G = G_;
    lc = t % CPR;
    r0 = (t / CPR) * RPT;
    sigma = BN % G;
    if (t < 4 * CPR) {  // entry (j, chunk): four cos or sin values of one chunk
      const int j = t / CPR, ch = t % CPR;
      float cs[4], sn[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) angle_cs(BN - BN / G, inv.v[8 * ch + 4 * (j & 1) + e], cs[e], sn[e]);
      tab.v[j][ch] = j < 2 ? make_float4(cs[0], cs[1], cs[2], cs[3]) : make_float4(sn[0], sn[1], sn[2], sn[3]);
    }
    const int J = j_first + r0;
    rho = J % G;
    const int n0 = corr_n(J, G);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float ca, sa, cb, sb;
      angle_cs(n0, inv.v[8 * lc + 2 * w], ca, sa);
      angle_cs(n0, inv.v[8 * lc + 2 * w + 1], cb, sb);
      bc[w] = make_float2(ca, cb);
      bs[w] = make_float2(sa, sb);
      angle_cs(1, inv.v[8 * lc + 2 * w], ca, sa);
      angle_cs(1, inv.v[8 * lc + 2 * w + 1], cb, sb);
      c1[w] = make_float2(ca, cb);
      s1[w] = make_float2(sa, sb);
    }
    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
  }

  // Rotate this thread's rows of one K tile (shared address of its first
  // byte), then advance the first-row rotation to the next key tile.
  __device__ __forceinline__ void rotate_tile(uint32_t tile, const KCorrTable &tab) {
    float2 c[4], s[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      c[w] = bc[w];
      s[w] = bs[w];
    }
    int rr = rho;  // key index of the current row, mod G
    auto addr_a = [&](int row) { return tile + row * 128 + ((lc ^ (row & 7)) << 4); };
    auto addr_b = [&](int row) {
      return D == 128 ? tile + HALF_BYTES + row * 128 + ((lc ^ (row & 7)) << 4)
                      : tile + row * 128 + (((lc + 4) ^ (row & 7)) << 4);
    };
    // row m + 1 is read before row m is written back, so each row's
    // shared-memory latency overlaps the previous row's arithmetic
    uint4 na = lds128(addr_a(r0)), nb = lds128(addr_b(r0));
#pragma unroll 1
    for (int m = 0; m < RPT; ++m) {
      const int row = r0 + m;
      uint4 xa = na, xb = nb;
      if (m + 1 < RPT) {
        na = lds128(addr_a(row + 1));
        nb = lds128(addr_b(row + 1));
      }
      uint32_t *ua = reinterpret_cast<uint32_t *>(&xa), *ub = reinterpret_cast<uint32_t *>(&xb);
      // R(-n) (a, b) = (a cos + b sin, b cos - a sin)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float2 fa = bf2_f2(ua[w]), fb = bf2_f2(ub[w]);
        ua[w] = f2_bf2(__ffma2_rn(fa, c[w], __fmul2_rn(fb, s[w])));
        ub[w] = f2_bf2(__ffma2_rn(fb, c[w], __fmul2_rn(neg2(fa), s[w])));
      }
      sts128(addr_a(row), xa);
      sts128(addr_b(row), xb);
      if (m + 1 < RPT) {
        if (rr + 1 == G) {
          rr = 0;  // the next key starts a group: n unchanged
        } else {
          ++rr;
#pragma unroll
          for (int w = 0; w < 4; ++w) compose2(c[w], s[w], c1[w], s1[w]);
        }
      }
    }
    // next tile: the first row advances by R(BN - b), and by R(-1) more when
    // the key index's residue carries past G
    const float4 tc0 = tab.v[0][lc], tc1 = tab.v[1][lc], ts0 = tab.v[2][lc], ts1 = tab.v[3][lc];
    const float2 dc[4] = {make_float2(tc0.x, tc0.y), make_float2(tc0.z, tc0.w), make_float2(tc1.x, tc1.y),
                          make_float2(tc1.z, tc1.w)};
    const float2 ds[4] = {make_float2(ts0.x, ts0.y), make_float2(ts0.z, ts0.w), make_float2(ts1.x, ts1.y),
                          make_float2(ts1.z, ts1.w)};
    const bool carry = rho + sigma >= G;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      compose2(bc[w], bs[w], dc[w], ds[w]);
      if (carry) compose2(bc[w], bs[w], c1[w], neg2(s1[w]));
    }
    rho += sigma - (carry ? G : 0);
  }

  // The role: every visit's K tile passes through here (stage v % NSTAGE,
  // in visit order); the grouped visits' tiles, the last n_grp visits on key
  // tiles in ascending order, are rotated, and each tile is then made visible
  // to the tensor core and released to the MMA issuer.
  __device__ __forceinline__ void run(int n_all, int n_grp, uint32_t kring, int stage_bytes, uint64_t *bar_kf,
                                      uint64_t *bar_kr, const KCorrTable &tab, volatile int *abort_flag,
                                      int *err) {
    for (int v = 0; v < n_all; ++v) {
      const int st = v % NSTAGE;
      if (!__all_sync(0xffffffffu, wait_b(&bar_kf[st], (v / NSTAGE) & 1, abort_flag, err, ERR_TIMEOUT_KCORR)))
        break;
      if (v >= n_all - n_grp) {
        rotate_tile(kring + st * stage_bytes, tab);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      mbar_arrive(&bar_kr[st]);
    }
  }
};

// ------------------------------------------------------------------ kernels
// One query head per CTA (odd GQA groups), 384 threads in 3 warpgroups:
//   warps 0-3   softmax / correction / epilogue: thread r owns query row r and
//               TMEM lane r; also rotates the query tile into grouped
//               positions once (R(f(i) - i) into the Q_g buffer).
//   warp 4      TMA producer of Q and K tiles (128 rows x D bf16, SWIZZLE_128B
//               boxes of 64 columns).
//   warp 5      TMEM allocator and the single-thread tcgen05.mma issuer:
//               S = Q K^T (SS form) into a double-buffered TMEM S, then
//               O += P V with P read from TMEM (TS form).
//   warp 6      TMA producer of V tiles.   (warp 7 idle)
//   warps 8-11  key correction: each grouped visit's K tile rotated in place.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,256+D) (fp32, lane = row);
// P (bf16 pairs) overwrites the first 64 columns of its S buffer.
template <int D>
__global__ void __launch_bounds__(P1_THREADS, 1)
bifocal_prefill_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                       const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mKg,
                       const __grid_constant__ Params p, const __grid_constant__ InvFreq inv) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_qg, bar_kf[P1_NKS], bar_kr[P1_NKS], bar_ke[P1_NKS], bar_vf[NVS],
      bar_ve[NVS], bar_sf[2], bar_pr[2], bar_od, bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ KCorrTable kctab;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item (uniform across the CTA; invalid items exit before any barrier)
  using GG = Geo<D>;
  constexpr int OFF_K1 = GG::P1_OFF_K;
  constexpr int OFF_V1 = GG::P1_OFF_V;
  const int s = blockIdx.z, h = blockIdx.y;
  const int a = p.cu[s];                // first query token
  const int L = p.cu[s + 1] - a;        // queries
  const int ak = p.cu_k[s];             // first key token
  const int Lk = p.cu_k[s + 1] - ak;    // keys: the sequence's current length
  if (L <= 0 || a < 0 || a + L > p.T || Lk < L || ak < 0 || ak + Lk > p.Tk) return;
  const int nqt = (L + BM - 1) / BM;
  if ((int)blockIdx.x >= nqt) return;
  Tile t;
  t.L = L;
  t.qt = nqt - 1 - (int)blockIdx.x;  // heaviest query tiles launch first
  t.i0 = t.qt * BM;
  t.i1 = min(t.i0 + BM - 1, L - 1);
  t.Lk = Lk;
  t.off = Lk - L;
  t.W = p.window;
  t.G = p.plain ? 1 : (int)group_size(Lk, p.w_pre);
  t.bif = t.G > 1;
  const int kvh = h / (p.Hq / p.Hkv);
  const VisitPlan pl = make_plan(t, p.w0);
  const bool need_qg = pl.n_grp > 0;
  const bool kcorr = need_qg && !p.kg_pre;  // grouped K tiles rotated in this CTA

  const uint32_t sbase = (su32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (sbase - su32(smem_raw));

  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_qg, 128);
    for (int i = 0; i < P1_NKS; ++i) {
      mbar_init(&bar_kf[i], 1);
      mbar_init(&bar_kr[i], 128);
      mbar_init(&bar_ke[i], 1);
    }
    for (int i = 0; i < NVS; ++i) { mbar_init(&bar_vf[i], 1); mbar_init(&bar_ve[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bar_sf[i], 1); mbar_init(&bar_pr[i], 128); }
    mbar_init(&bar_od, 1);
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 4 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mQ) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mK) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mV) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mKg) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  const int tok_q0 = a + t.i0;
  if (warp >= 8) {
    // ================= key correction (warps 8-11) =================
    regs_dec<P1_REG_KCORR>();
    if (kcorr) {
      KeyCorrection<D, P1_NKS> kc;
      kc.init(threadIdx.x - 256, pl.g_begin * BN, t.G, inv, kctab, 1);
      kc.run(pl.n_all, pl.n_grp, sbase + OFF_K1, GG::TB, bar_kf, bar_kr, kctab, &abort_flag, p.err);
    }
  } else if (warp >= 4) {
    regs_dec<P1_REG_IO>();
    if (warp == 4 && lane == 0) {
      // ================= producer: Q, then K tiles in visit order =================
      // (K and V are kept in L2 ahead of the query tile, read once)
      const uint64_t pol_kv = l2_evict_last(), pol_q = l2_evict_first();
      mbar_expect_tx(&bar_q, GG::TB);
      for (int hf = 0; hf < GG::NH; ++hf)
        tma_load_hint(&mQ, &bar_q, sbase + OFF_Q + hf * HALF_BYTES, 64 * hf, h, tok_q0, pol_q);
      int v = 0;
      for (; v < pl.n_all; ++v) {
        int kt;
        Visit vx;
        visit_at(t, pl, p.w0, v, kt, vx);
        const int st = v % P1_NKS;
        if (v >= P1_NKS &&
            !wait_b(&bar_ke[st], ((v / P1_NKS) - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_PRODUCER))
          break;
        const CUtensorMap *m = (vx.grp && p.kg_pre) ? &mKg : &mK;
        const uint32_t dst = sbase + OFF_K1 + st * GG::TB;
        mbar_expect_tx(&bar_kf[st], GG::TB);
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load_hint(m, &bar_kf[st], dst + hf * HALF_BYTES, 64 * hf, kvh, ak + kt * BN, pol_kv);
      }
      // drain: every load issued must land before the CTA may exit
      for (int u = max(0, v - P1_NKS); u < v; ++u)
        wait_drain(&bar_kf[u % P1_NKS], (u / P1_NKS) & 1, p.err, ERR_TIMEOUT_PRODUCER);
      wait_drain(&bar_q, 0, p.err, ERR_TIMEOUT_PRODUCER);
    } else if (warp == 6 && lane == 0) {
      // ================= producer: V tiles in visit order =================
      const uint64_t pol_kv = l2_evict_last();
      int v = 0;
      for (; v < pl.n_all; ++v) {
        int kt;
        Visit vx;
        visit_at(t, pl, p.w0, v, kt, vx);
        const int st = v % NVS;
        if (v >= NVS && !wait_b(&bar_ve[st], ((v / NVS) - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_PRODUCER))
          break;
        const uint32_t dst = sbase + OFF_V1 + st * GG::TB;
        mbar_expect_tx(&bar_vf[st], GG::TB);
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load_hint(&mV, &bar_vf[st], dst + hf * HALF_BYTES, 64 * hf, kvh, ak + kt * BN, pol_kv);
      }
      for (int u = max(0, v - NVS); u < v; ++u) wait_drain(&bar_vf[u % NVS], (u / NVS) & 1, p.err, ERR_TIMEOUT_PRODUCER);
    } else if (warp == 5 && lane == 0) {
      // ================= MMA issuer (one thread) =================
      bool ok = wait_b(&bar_q, 0, &abort_flag, p.err, ERR_TIMEOUT_MMA);
      bool qg_seen = false;
      int v = 0;
      // descriptor halves: the start address field (addr >> 4, 14 bits) of
      // every stage and k-step stays below 2^14, so a stage or a k-step adds
      // to the low half only; the high halves are fixed
      const uint64_t vd0 = desc_mn_sw128(sbase + OFF_V1, HALF_BYTES);
      const uint32_t v0lo = (uint32_t)vd0, vhi = (uint32_t)(vd0 >> 32);
      const uint64_t kd0 = desc_k_sw128(sbase + OFF_K1);
      const uint32_t k0lo = (uint32_t)kd0, dhi = (uint32_t)(kd0 >> 32);
      const uint32_t qlo_b = (uint32_t)desc_k_sw128(sbase + OFF_Q), qlo_g = (uint32_t)desc_k_sw128(sbase + GG::P1_OFF_QG);
      auto issue_pv = [&](int u) -> bool {
        const int vs_ = u % NVS;
        if (!wait_b(&bar_vf[vs_], (u / NVS) & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA)) return false;
        if (!wait_b(&bar_pr[u & 1], (u >> 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint32_t vlo = v0lo + (uint32_t)vs_ * (uint32_t)(GG::TB >> 4);
        const uint32_t pcol = tmem + (uint32_t)((u & 1) * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts_lh(tmem + COL_O, pcol + kk * 8, vlo + kk * 128, vhi, GG::IDESC_PV, (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bar_ve[vs_]);
        umma_commit(&bar_od);
        return true;
      };
      for (; v < pl.n_all && ok; ++v) {
        int kt;
        Visit vx;
        visit_at(t, pl, p.w0, v, kt, vx);
        if (vx.grp && !qg_seen) {
          if (!(ok = wait_b(&bar_qg, 0, &abort_flag, p.err, ERR_TIMEOUT_MMA))) break;
          qg_seen = true;
        }
        const int st = v % P1_NKS;
        // with the key correction running, every K tile passes through it
        // (the grouped ones rotated) before the MMA reads it
        uint64_t *kready = kcorr ? &bar_kr[st] : &bar_kf[st];
        if (!(ok = wait_b(kready, (v / P1_NKS) & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA))) break;
        tc_fence_after();
        const uint32_t qlo = vx.grp ? qlo_g : qlo_b;
        const uint32_t kdlo = k0lo + (uint32_t)st * (uint32_t)(GG::TB >> 4);
        const uint32_t scol = tmem + (uint32_t)((v & 1) * 128);
#pragma unroll
        for (int kk = 0; kk < GG::KSTEPS; ++kk) {
          const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
          umma_ss_lh(scol, qlo + off, dhi, kdlo + off, dhi, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar_sf[v & 1]);
        umma_commit(&bar_ke[st]);
        if (v > 0 && !(ok = issue_pv(v - 1))) break;
      }
      if (ok && v > 0) issue_pv(v - 1);
      // all MMAs issued so far must finish before TMEM is released
      umma_commit(&bar_drain);
      wait_drain(&bar_drain, 0, p.err, ERR_TIMEOUT_MMA);
    }
  } else {
    // ================= softmax warpgroup (warps 0-3) =================
    regs_inc<P1_REG_SOFTMAX>();
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int i = t.i0 + r;
    bool ok = true;
    if (need_qg) {
      // rotate the query tile into grouped positions: Q_g = R(f(i) - i) Q~
      ok = __all_sync(0xffffffffu, wait_b(&bar_q, 0, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
      if (ok) {
        // pair k = (element k, element k + D/2): D = 128, chunk u of box 0
        // and the same chunk of box 1; D = 64, logical chunk lc and lc + 4 of
        // the one 128-byte row
        for (int kk = 0; kk < (D == 128 ? 8 : 4); ++kk) {
          const int u = r + 128 * kk;
          const int row = D == 128 ? u >> 3 : u >> 2;
          const int lc = D == 128 ? (u & 7) ^ (row & 7) : u & 3;  // logical 8-column group
          const int n = corr_n(t.off + min(t.i0 + row, L - 1), t.G);
          const int oa = D == 128 ? u * 16 : row * 128 + ((lc ^ (row & 7)) << 4);
          const int ob = D == 128 ? HALF_BYTES + u * 16 : row * 128 + (((lc + 4) ^ (row & 7)) << 4);
          uint4 xa = *reinterpret_cast<const uint4 *>(gbase + OFF_Q + oa);
          uint4 xb = *reinterpret_cast<const uint4 *>(gbase + OFF_Q + ob);
          uint32_t *pa = reinterpret_cast<uint32_t *>(&xa), *pb = reinterpret_cast<uint32_t *>(&xb);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pa[e2]));
            float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pb[e2]));
            float c0, s0, c1, s1;
            angle_cs(n, inv.v[lc * 8 + 2 * e2], c0, s0);
            angle_cs(n, inv.v[lc * 8 + 2 * e2 + 1], c1, s1);
            rot_back(fa.x, fb.x, c0, s0);
            rot_back(fa.y, fb.y, c1, s1);
            __nv_bfloat162 ra = __floats2bfloat162_rn(fa.x, fa.y);
            __nv_bfloat162 rb = __floats2bfloat162_rn(fb.x, fb.y);
            pa[e2] = *reinterpret_cast<uint32_t *>(&ra);
            pb[e2] = *reinterpret_cast<uint32_t *>(&rb);
          }
          *reinterpret_cast<uint4 *>(gbase + GG::P1_OFF_QG + oa) = xa;
          *reinterpret_cast<uint4 *>(gbase + GG::P1_OFF_QG + ob) = xb;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bar_qg);
    }

    float m_run = -INFINITY, l_run = 0.f;
    int v = 0;
    for (; v < pl.n_all && ok; ++v) {
      int kt;
      Visit vx;
      visit_at(t, pl, p.w0, v, kt, vx);
      const int dc = t.off + i - kt * BN;  // column c has distance dc - c
      {
        const int b = v & 1;
        ok = __all_sync(0xffffffffu, wait_b(&bar_sf[b], (v >> 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
        if (!ok) break;
        tc_fence_after();
        const uint32_t scol = tmem + lane_base + (uint32_t)(b * 128);
        float sv[128];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(scol + 0, r0);
          tmem_ld32(scol + 32, r1);
          tmem_ld32(scol + 64, r2);
          tmem_ld32(scol + 96, r3);
          tmem_wait_ld_regs(r0);
          tmem_wait_ld_regs(r1);
          tmem_wait_ld_regs(r2);
          tmem_wait_ld_regs(r3);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[e] = __uint_as_float(r0[e]);
            sv[32 + e] = __uint_as_float(r1[e]);
            sv[64 + e] = __uint_as_float(r2[e]);
            sv[96 + e] = __uint_as_float(r3[e]);
          }
        }
        if (vx.mask) {
          const int cmin = max(0, dc - vx.hi);
          const int cmax = min(BN - 1, dc - vx.lo);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < cmin || c > cmax) sv[c] = -INFINITY;
        }
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) mt = fmaxf(mt, sv[c]);
        mt *= p.sl2;
        const float m_new = fmaxf(m_run, mt);
        const bool need = (m_run != -INFINITY) && (m_new > m_run + 8.0f);
        if (m_run == -INFINITY) m_run = m_new;
        if (__any_sync(0xffffffffu, need)) {
          // O holds PV of visits < v; PV_{v-1} may still run: wait for it
          ok = __all_sync(0xffffffffu, wait_b(&bar_od, (v - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
          if (!ok) break;
          tc_fence_after();
          const float f = need ? ex2(m_run - m_new) : 1.0f;
          if (need) {
            l_run *= f;
            m_run = m_new;
          }
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t rr[32];
            tmem_ld32(tmem + lane_base + COL_O + c4 * 32, rr);
            tmem_wait_ld_regs(rr);
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * f);
            tmem_st32(tmem + lane_base + COL_O + c4 * 32, rr);
          }
          tmem_wait_st();
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float lsum = 0.f;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float p0 = ex2(fmaf(sv[h2 * 64 + 2 * e], p.sl2, -m_use));
            const float p1 = ex2(fmaf(sv[h2 * 64 + 2 * e + 1], p.sl2, -m_use));
            lsum += p0 + p1;
            __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<uint32_t *>(&pb);
          }
          tmem_st32(scol + h2 * 32, pk);
        }
        l_run += lsum;
        tmem_wait_st();
        // the last visit: make sure PV_{v-1} is done so that exactly one PV
        // (this visit's) is outstanding when the epilogue waits
        const bool last = v == pl.n_all - 1;
        if (last && v > 0) {
          ok = __all_sync(0xffffffffu, wait_b(&bar_od, (v - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
        }
        tc_fence_before();
        mbar_arrive(&bar_pr[b]);
      }
    }
    // ---- epilogue: O / l -> bf16, LSE
    if (ok && v > 0) ok = __all_sync(0xffffffffu, wait_b(&bar_od, (v - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
    if (ok) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      const bool row_ok = i < L;
      const uint64_t pol_o = l2_evict_first();  // written once, never read here
      __nv_bfloat16 *orow = p.out + ((size_t)(tok_q0 + r) * p.Hq + h) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + COL_O + c4 * 32, rr);
        tmem_wait_ld_regs(rr);
        if (row_ok) {
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
            uint4 o4;
            uint32_t *po = reinterpret_cast<uint32_t *>(&o4);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              __nv_bfloat162 ob = __floats2bfloat162_rn(__uint_as_float(rr[e8 * 8 + 2 * e2]) * inv_l,
                                                        __uint_as_float(rr[e8 * 8 + 2 * e2 + 1]) * inv_l);
              po[e2] = *reinterpret_cast<uint32_t *>(&ob);
            }
            stg128_hint(orow + c4 * 32 + e8 * 8, o4, pol_o);
          }
        }
      }
      if (row_ok && p.lse != nullptr)
        p.lse[(size_t)h * p.T + tok_q0 + r] =
            (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ---- teardown: every role has drained its own asynchronous work
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// Ablation of the key correction (JL_FLAG_PREROTATE_K): grouped keys
// K_g = R(f(j) - j) K~ for every token of sequences with G > 1, written once
// per key into the workspace (all kv heads of a token share the angles), and
// TMA-loaded by the grouped visits instead of being rotated in the tile.
__global__ void __launch_bounds__(256)
prerotate_k_kernel(const __nv_bfloat16 *__restrict__ k, __nv_bfloat16 *__restrict__ kg, int D,
                   const int32_t *__restrict__ cu, int batch, int T, int Hkv, long long w_pre,
                   const __grid_constant__ InvFreq inv) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_tok = D / 16;  // threads per token, 8 pairs each
  if (gid >= (long long)T * per_tok) return;
  const int tok = (int)(gid / per_tok), cg = (int)(gid % per_tok);  // pairs k = 8cg .. 8cg+7
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= tok) lo = mid; else hi = mid;
  }
  const int a = cu[lo], L = cu[lo + 1] - a, pos = tok - a;
  if (L <= 0 || pos < 0 || pos >= L) return;
  const int G = (int)group_size(L, w_pre);
  if (G <= 1) return;  // never read: sequences with G = 1 have no grouped visit
  const int n = corr_n(pos, G);
  float cs[8], sn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) angle_cs(n, inv.v[cg * 8 + e], cs[e], sn[e]);
  for (int hh = 0; hh < Hkv; ++hh) {
    const size_t base = ((size_t)tok * Hkv + hh) * D + cg * 8;
    uint4 xa = *reinterpret_cast<const uint4 *>(k + base);
    uint4 xb = *reinterpret_cast<const uint4 *>(k + base + D / 2);
    uint32_t *pa = reinterpret_cast<uint32_t *>(&xa), *pb = reinterpret_cast<uint32_t *>(&xb);
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pa[e2]));
      float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pb[e2]));
      rot_back(fa.x, fb.x, cs[2 * e2], sn[2 * e2]);
      rot_back(fa.y, fb.y, cs[2 * e2 + 1], sn[2 * e2 + 1]);
      __nv_bfloat162 ra = __floats2bfloat162_rn(fa.x, fa.y);
      __nv_bfloat162 rb = __floats2bfloat162_rn(fb.x, fb.y);
      pa[e2] = *reinterpret_cast<uint32_t *>(&ra);
      pb[e2] = *reinterpret_cast<uint32_t *>(&rb);
    }
    *reinterpret_cast<uint4 *>(kg + base) = xa;
    *reinterpret_cast<uint4 *>(kg + base + D / 2) = xb;
  }
}


// packed fp32 pairs (sm_100 f32x2): one instruction for two lanes of data
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// ===========================================================================
// Two heads per CTA.
//
// The CTA takes one 128-row query tile of two query heads of the same GQA
// group: both read the same K/V tiles (loaded, and for grouped visits
// rotated, once), and two softmax warpgroups ping-pong against one MMA warp,
// so the tensor core always has the other head's QK or PV to run while a
// softmax warpgroup works.  512 threads, 4 warpgroups:
//   warps 0-3 / 4-7  softmax of head A / head B (thread = row = TMEM lane);
//                    the row's 128 scores are read from TMEM once and stay
//                    in registers (setmaxnreg gives these warpgroups the
//                    registers the other two do not need)
//   warps 8-11       key correction: each grouped visit's K tile rotated in
//                    place, R(f(j) - j), before its QK products
//   warp 12          TMA producers: lane 0 streams Q and K tiles, lane 1 V tiles
//   warp 13          TMEM allocator and tcgen05.mma issuer   (warps 14-15 idle)
// TMEM: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [256+D,256+2D).
// Visit order: every grouped visit (ascending key tile), then every base
// visit.  The query tiles are rotated in place into grouped positions for
// the first phase and re-loaded by TMA for the second.
// ===========================================================================
template <int D>
__global__ void __launch_bounds__(P2_THREADS, 1)
bifocal_prefill2_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                        const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mKg,
                        const __grid_constant__ Params p, const __grid_constant__ InvFreq inv) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_qg[2], bar_kf[P2_NKS], bar_kr[P2_NKS],
      bar_ke[P2_NKS], bar_vf[P2_NVS], bar_ve[P2_NVS], bar_sf[2], bar_pr[2], bar_ph[2], bar_od[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ KCorrTable kctab;

  using GG = Geo<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.z;
  // x enumerates (query tile, head pair of the kv head) with the head pair
  // fastest, so the CTAs of all head pairs of one kv head run side by side
  // and sweep the same K and V tiles at the same time (shared in L2)
  const int ppk = p.Hq / p.Hkv / 2;          // head pairs per kv head
  const int qx = (int)blockIdx.x / ppk;      // query-tile index (heaviest first)
  const int hA = 2 * ((int)blockIdx.y * ppk + (int)blockIdx.x % ppk);  // heads hA, hA + 1
  const int a = p.cu[s];                // first query token
  const int L = p.cu[s + 1] - a;        // queries
  const int ak = p.cu_k[s];             // first key token
  const int Lk = p.cu_k[s + 1] - ak;    // keys: the sequence's current length
  if (L <= 0 || a < 0 || a + L > p.T || Lk < L || ak < 0 || ak + Lk > p.Tk) return;
  const int nqt = (L + BM - 1) / BM;
  if (qx >= nqt) return;
  Tile t;
  t.L = L;
  t.qt = nqt - 1 - qx;
  t.i0 = t.qt * BM;
  t.i1 = min(t.i0 + BM - 1, L - 1);
  t.Lk = Lk;
  t.off = Lk - L;
  t.W = p.window;
  t.G = p.plain ? 1 : (int)group_size(Lk, p.w_pre);
  t.bif = t.G > 1;
  const int kvh = hA / (p.Hq / p.Hkv);
  // visits: grouped ones first
  const VisitPlan pl = make_plan(t, p.w0);
  const int n_grp = pl.n_grp, n_all = pl.n_all;
  const int n_base = n_all - n_grp;            // base visits first, then grouped
  const bool kcorr = n_grp > 0 && !p.kg_pre;  // grouped K tiles rotated in this CTA

  const uint32_t sbase = (su32(smem_raw) + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (sbase - su32(smem_raw));

  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_qg[0], 128);
    mbar_init(&bar_qg[1], 128);
    for (int i = 0; i < P2_NKS; ++i) {
      mbar_init(&bar_kf[i], 1);
      mbar_init(&bar_kr[i], 128);
      mbar_init(&bar_ke[i], 1);
    }
    for (int i = 0; i < P2_NVS; ++i) { mbar_init(&bar_vf[i], 1); mbar_init(&bar_ve[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_sf[i], 1);
      mbar_init(&bar_pr[i], 128);
      mbar_init(&bar_ph[i], 128);
      mbar_init(&bar_od[i], 1);
    }
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 13) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 12 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mQ) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mK) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mV) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mKg) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int tok_q0 = a + t.i0;
  if (warp >= 12) {
    regs_dec<P2_REG_IO>();
    if (warp == 12 && lane == 0) {
      // ================= producer: Q, then K tiles in visit order.  K and V
      // tiles are read by every CTA of the kv head: kept in L2 ahead of the
      // query tiles, which one CTA reads once.
      const uint64_t pol_kv = l2_evict_last(), pol_q = l2_evict_first();
      mbar_expect_tx(&bar_q, 2 * GG::TB);
      for (int x = 0; x < 2; ++x)
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load_hint(&mQ, &bar_q, sbase + P2_OFF_Q + x * GG::TB + hf * HALF_BYTES, 64 * hf, hA + x, tok_q0,
                        pol_q);
      bool ok = true;
      int v = 0;
      for (; ok && v < n_all;) {
        int kt;
        Visit vv;
        visit_at(t, pl, p.w0, v, kt, vv);
        const int st = v % P2_NKS;
        if (v >= P2_NKS && !(ok = wait_b(&bar_ke[st], ((v / P2_NKS) - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_PRODUCER)))
          break;
        const CUtensorMap *m = (vv.grp && p.kg_pre) ? &mKg : &mK;
        const uint32_t dst = sbase + GG::OFF_K + st * GG::TB;
        mbar_expect_tx(&bar_kf[st], GG::TB);
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load_hint(m, &bar_kf[st], dst + hf * HALF_BYTES, 64 * hf, kvh, ak + kt * BN, pol_kv);
        ++v;
      }
      for (int u = max(0, v - P2_NKS); u < v; ++u)
        wait_drain(&bar_kf[u % P2_NKS], (u / P2_NKS) & 1, p.err, ERR_TIMEOUT_PRODUCER);
      wait_drain(&bar_q, 0, p.err, ERR_TIMEOUT_PRODUCER);
    } else if (warp == 12 && lane == 1) {
      // ================= producer: V tiles in visit order
      const uint64_t pol_kv = l2_evict_last();
      bool ok = true;
      int v = 0;
      for (; ok && v < n_all;) {
        int kt;
        Visit vv;
        visit_at(t, pl, p.w0, v, kt, vv);
        const int st = v % P2_NVS;
        if (v >= P2_NVS && !(ok = wait_b(&bar_ve[st], ((v / P2_NVS) - 1) & 1, &abort_flag, p.err, ERR_TIMEOUT_PRODUCER)))
          break;
        const uint32_t dst = sbase + GG::OFF_V + st * GG::TB;
        mbar_expect_tx(&bar_vf[st], GG::TB);
        for (int hf = 0; hf < GG::NH; ++hf)
          tma_load_hint(&mV, &bar_vf[st], dst + hf * HALF_BYTES, 64 * hf, kvh, ak + kt * BN, pol_kv);
        ++v;
      }
      for (int u = max(0, v - P2_NVS); u < v; ++u)
        wait_drain(&bar_vf[u % P2_NVS], (u / P2_NVS) & 1, p.err, ERR_TIMEOUT_PRODUCER);
    } else if (warp == 13 && lane == 0) {
      // ================= MMA issuer (one thread), fixed order:
      //   QK_A(0) QK_B(0), then per visit v: PV_A(v) QK_A(v+1) PV_B(v) QK_B(v+1)
      // so that each softmax warpgroup's next S is computed while the other
      // head's PV runs.  S_x is reused by QK_x(v+1) only after PV_x(v) (which
      // read P_x(v) from it) has been issued.
      bool ok = wait_b(&bar_q, 0, &abort_flag, p.err, ERR_TIMEOUT_MMA);
      // descriptor halves: the start address field (addr >> 4, 14 bits) of
      // every stage and k-step stays below 2^14, so a stage or a k-step adds
      // to the low half only; the high halves are fixed
      const uint64_t qd0 = desc_k_sw128(sbase + P2_OFF_Q), vd0 = desc_mn_sw128(sbase + GG::OFF_V, HALF_BYTES);
      const uint32_t q0lo = (uint32_t)qd0, q1lo = q0lo + (uint32_t)(GG::TB >> 4), dhi = (uint32_t)(qd0 >> 32);
      const uint32_t k0lo = (uint32_t)desc_k_sw128(sbase + GG::OFF_K);
      const uint32_t v0lo = (uint32_t)vd0, vhi = (uint32_t)(vd0 >> 32);
      auto issue_qk = [&](int x, int v) -> bool {
        // the first grouped QK of a head reads its query tile rotated in
        // place by that head's softmax warpgroup
        if (v == n_base && n_grp > 0 && !wait_b(&bar_qg[x], 0, &abort_flag, p.err, ERR_TIMEOUT_MMA)) return false;
        // a grouped K tile is read once the key correction has rotated it
        // (with the key correction running, every K tile passes through it)
        if (x == 0) {
          uint64_t *kready = kcorr ? &bar_kr[v % P2_NKS] : &bar_kf[v % P2_NKS];
          if (!wait_b(kready, (v / P2_NKS) & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA)) return false;
        }
        tc_fence_after();
        const uint32_t scol = tmem + (uint32_t)(x * 128);
        const uint32_t qlo = x ? q1lo : q0lo, kdlo = k0lo + (uint32_t)(v % P2_NKS) * (uint32_t)(GG::TB >> 4);
        umma_ss_lhc<0>(scol, qlo, dhi, kdlo, dhi, IDESC_QK);
#pragma unroll
        for (int kk = 1; kk < GG::KSTEPS; ++kk) {
          const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
          umma_ss_lhc<1>(scol, qlo + off, dhi, kdlo + off, dhi, IDESC_QK);
        }
        umma_commit(&bar_sf[x]);
        if (x == 1) umma_commit(&bar_ke[v % P2_NKS]);  // both heads' QK issued
        return true;
      };
      auto issue_pv = [&](int x, int v) -> bool {
        // P arrives in two halves (keys 0-63, then 64-127): the first half
        // of PV runs while the softmax finishes the second
        if (!wait_b(&bar_ph[x], v & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA)) return false;
        // both heads read the same V stage: head A's issue waited for it
        if (x == 0 && !wait_b(&bar_vf[v % P2_NVS], (v / P2_NVS) & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA))
          return false;
        tc_fence_after();
        const uint32_t pcol = tmem + (uint32_t)(x * 128);
        const uint32_t ocol = tmem + COL_O + (uint32_t)(x * D);
        const uint32_t vlo = v0lo + (uint32_t)(v % P2_NVS) * (uint32_t)(GG::TB >> 4);
        umma_ts_lh(ocol, pcol, vlo, vhi, GG::IDESC_PV, v > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 4; ++kk) umma_ts_lhc<1>(ocol, pcol + kk * 8, vlo + kk * 128, vhi, GG::IDESC_PV);
        if (!wait_b(&bar_pr[x], v & 1, &abort_flag, p.err, ERR_TIMEOUT_MMA)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 4; kk < 8; ++kk) umma_ts_lhc<1>(ocol, pcol + kk * 8, vlo + kk * 128, vhi, GG::IDESC_PV);
        if (v == n_all - 1) umma_commit(&bar_od[x]);  // the epilogue's wait: the last PV
        if (x == 1) umma_commit(&bar_ve[v % P2_NVS]);
        return true;
      };
      if (ok && n_all > 0) ok = issue_qk(0, 0) && issue_qk(1, 0);
      for (int v = 0; ok && v < n_all; ++v) {
        ok = issue_pv(0, v);
        if (ok && v + 1 < n_all) ok = issue_qk(0, v + 1);
        if (ok) ok = issue_pv(1, v);
        if (ok && v + 1 < n_all) ok = issue_qk(1, v + 1);
      }
      umma_commit(&bar_drain);
      wait_drain(&bar_drain, 0, p.err, ERR_TIMEOUT_MMA);
    }
  } else if (warp >= 8) {
    // ================= key correction (warps 8-11)
    regs_dec<P2_REG_KCORR>();
    if (kcorr) {
      KeyCorrection<D, P2_NKS> kc;
      kc.init(threadIdx.x - 256, pl.g_begin * BN, t.G, inv, kctab, 1);
      kc.run(n_all, n_grp, sbase + GG::OFF_K, GG::TB, bar_kf, bar_kr, kctab, &abort_flag, p.err);
    }
  } else {
    // ================= softmax warpgroups (warps 0-3: head A, 4-7: head B)
    regs_inc<P2_REG_SOFTMAX>();
    const int hx = warp >> 2;
    const int r = threadIdx.x & 127;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t scol = tmem + lane_base + (uint32_t)(hx * 128);
    const uint32_t ocol = tmem + lane_base + COL_O + (uint32_t)(hx * D);
    const int i = t.i0 + r;
    const int h = hA + hx;
    bool ok = true;
    // rotate this head's query tile in place, Q_g = R(f(i) - i) Q~, once its
    // base-phase QK products are done (the S of its last base visit is ready)
    // or, with no base visit, once it has landed
    auto rotate_q = [&]() {
      uint8_t *qt = gbase + P2_OFF_Q + hx * GG::TB;
      // pair k = (element k, element k + D/2).  D = 128: chunk u of box 0
      // pairs with the same chunk of box 1.  D = 64: in the one 128-byte
      // row, logical chunk lc (elements 8 lc ..) pairs with chunk lc + 4.
      for (int kk = 0; kk < (D == 128 ? 8 : 4); ++kk) {
        const int u = r + 128 * kk;
        const int row = D == 128 ? u >> 3 : u >> 2;
        const int lc = D == 128 ? (u & 7) ^ (row & 7) : u & 3;
        const int n = corr_n(t.off + min(t.i0 + row, L - 1), t.G);
        uint4 *qa = reinterpret_cast<uint4 *>(D == 128 ? qt + u * 16 : qt + row * 128 + ((lc ^ (row & 7)) << 4));
        uint4 *qb = reinterpret_cast<uint4 *>(D == 128 ? qt + HALF_BYTES + u * 16
                                                       : qt + row * 128 + (((lc + 4) ^ (row & 7)) << 4));
        uint4 xa = *qa, xb = *qb;
        uint32_t *pa = reinterpret_cast<uint32_t *>(&xa), *pb = reinterpret_cast<uint32_t *>(&xb);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pa[e2]));
          float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pb[e2]));
          float c0, s0, c1, s1;
          angle_cs(n, inv.v[lc * 8 + 2 * e2], c0, s0);
          angle_cs(n, inv.v[lc * 8 + 2 * e2 + 1], c1, s1);
          rot_back(fa.x, fb.x, c0, s0);
          rot_back(fa.y, fb.y, c1, s1);
          __nv_bfloat162 ra = __floats2bfloat162_rn(fa.x, fa.y);
          __nv_bfloat162 rb = __floats2bfloat162_rn(fb.x, fb.y);
          pa[e2] = *reinterpret_cast<uint32_t *>(&ra);
          pb[e2] = *reinterpret_cast<uint32_t *>(&rb);
        }
        *qa = xa;
        *qb = xb;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bar_qg[hx]);
    };
    if (n_grp > 0 && n_base == 0) {
      ok = __all_sync(0xffffffffu, wait_b(&bar_q, 0, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
      rotate_q();
    }

    float m_run = -INFINITY, l_run = 0.f;
    int v = 0;
    for (; ok && v < n_all;) {
      int kt;
      Visit vv;
      visit_at(t, pl, p.w0, v, kt, vv);
      ok = __all_sync(0xffffffffu, wait_b(&bar_sf[hx], v & 1, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
      tc_fence_after();
      // the head's last base visit: its QK products (which read Q~) are done
      if (v == n_base - 1 && n_grp > 0) rotate_q();
      if (!ok) break;
      // columns c with distance dc - c outside [lo, hi] are masked; the
      // visit-uniform mask flag selects a specialisation without compares
      const int dc = t.off + i - kt * BN;  // row position minus the tile's first key
      const int cmin = vv.mask ? max(0, dc - vv.hi) : 0;
      const int cmax = vv.mask ? min(BN - 1, dc - vv.lo) : BN - 1;
      float2 l2a = make_float2(0.f, 0.f), l2b = make_float2(0.f, 0.f);
      auto visit_body = [&](auto masked) {
        constexpr bool MASKED = decltype(masked)::value;
        auto sel = [&](int c, uint32_t raw) -> float {
          if constexpr (MASKED) return (c < cmin || c > cmax) ? -INFINITY : __uint_as_float(raw);
          else return __uint_as_float(raw);
        };
        // one pass over TMEM: the four 32-column loads are in flight
        // together and the row's 128 scores stay in registers
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(scol + 0, r0);
        tmem_ld32(scol + 32, r1);
        tmem_ld32(scol + 64, r2);
        tmem_ld32(scol + 96, r3);
        tmem_wait_ld_regs(r0);
        tmem_wait_ld_regs(r1);
        tmem_wait_ld_regs(r2);
        tmem_wait_ld_regs(r3);
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          m4[0] = fmaxf(m4[0], sel(e, r0[e]));
          m4[1] = fmaxf(m4[1], sel(e + 32, r1[e]));
          m4[2] = fmaxf(m4[2], sel(e + 64, r2[e]));
          m4[3] = fmaxf(m4[3], sel(e + 96, r3[e]));
        }
        const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.sl2;
        const float m_new = fmaxf(m_run, mt);
        const bool need = (m_run != -INFINITY) && (m_new > m_run + 8.0f);
        if (m_run == -INFINITY) m_run = m_new;
        if (__any_sync(0xffffffffu, need)) {
          // O_x holds PV of visits < v, all complete: QK_x(v) was issued after
          // PV_x(v-1) and the S_x commit covers it
          const float f = need ? ex2(m_run - m_new) : 1.0f;
          if (need) {
            l_run *= f;
            m_run = m_new;
          }
#pragma unroll
          for (int c4 = 0; c4 < D / 16; ++c4) {
            uint32_t rr[16];
            tmem_ld16(ocol + c4 * 16, rr);
#pragma unroll
            for (int e = 0; e < 16; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * f);
            tmem_st16(ocol + c4 * 16, rr);
          }
          tmem_wait_st();
        }
        // P = exp2(s * scale - m) as bf16 pairs: the 32 columns from c0 land
        // on TMEM columns c0 / 2 .. c0 / 2 + 15 (already read)
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        auto emit = [&](const uint32_t(&rr)[32], int c0) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = c0 + 2 * e;
            const float x0 = sel(c, rr[2 * e]);
            const float x1 = sel(c + 1, rr[2 * e + 1]);
            const float2 a2 = ffma2(make_float2(x0, x1), make_float2(p.sl2, p.sl2), make_float2(-m_use, -m_use));
            const float p0 = ex2(a2.x);
            const float p1 = ex2(a2.y);
            if (e & 1) l2b = fadd2(l2b, make_float2(p0, p1));
            else l2a = fadd2(l2a, make_float2(p0, p1));
            __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<uint32_t *>(&pb);
          }
          tmem_st16(scol + (c0 >> 1), pk);
        };
        emit(r0, 0);
        emit(r1, 32);
        // keys 0-63 of P are in TMEM: the first half of PV may start
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_ph[hx]);
        emit(r2, 64);
        emit(r3, 96);
      };
      if (vv.mask)
        visit_body(std::true_type{});
      else
        visit_body(std::false_type{});
      l_run += (l2a.x + l2a.y) + (l2b.x + l2b.y);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_pr[hx]);
      ++v;
    }
    // ---- epilogue: exactly one PV (the last) can be outstanding
    if (ok && v > 0) ok = __all_sync(0xffffffffu, wait_b(&bar_od[hx], 0, &abort_flag, p.err, ERR_TIMEOUT_SOFTMAX));
    if (ok) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      const bool row_ok = i < L;
      const uint64_t pol_o = l2_evict_first();  // written once, never read here
      __nv_bfloat16 *orow = p.out + ((size_t)(tok_q0 + r) * p.Hq + h) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t rr[32];
        tmem_ld32(ocol + c4 * 32, rr);
        tmem_wait_ld_regs(rr);
        if (row_ok) {
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
            uint4 o4;
            uint32_t *po = reinterpret_cast<uint32_t *>(&o4);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              __nv_bfloat162 ob = __floats2bfloat162_rn(__uint_as_float(rr[e8 * 8 + 2 * e2]) * inv_l,
                                                        __uint_as_float(rr[e8 * 8 + 2 * e2 + 1]) * inv_l);
              po[e2] = *reinterpret_cast<uint32_t *>(&ob);
            }
            stg128_hint(orow + c4 * 32 + e8 * 8, o4, pol_o);
          }
        }
      }
      if (row_ok && p.lse != nullptr)
        p.lse[(size_t)h * p.T + tok_q0 + r] =
            (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

}  // namespace tc

// ------------------------------------------------------------------ host
namespace {

// [T, H, D] bf16 viewed as a 3-D tensor (d, head, token); box 64 x 1 x 128.
bool make_map(CUtensorMap *m, const void *base, int T, int H, int D) {
  EncodeTiledFn enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)tc::BM};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Workspace: a 256-byte error word; with JL_FLAG_PREROTATE_K (the ablation of
// the in-tile key correction) also the grouped keys K_g, laid out like K.
size_t tc_prefill_workspace(int batch, int T_total, int Hq, int Hkv, int D, uint32_t flags) {
  (void)batch; (void)Hq;
  const bool pre = (flags & JL_FLAG_PREROTATE_K) != 0;
  return 256 + (pre ? a256((size_t)T_total * Hkv * D * 2) : 0);
}

cudaError_t launch_tc_prefill(const void *q, const void *k, const void *v, void *out, float *lse,
                              const int32_t *cu, const int32_t *cu_k, int batch, int T_total, int Tk,
                              int max_seqlen, int Hq, int Hkv, int D, long long w_pre, int w0, int window,
                              const InvFreq &inv, int plain, uint32_t flags, void *ws, size_t ws_bytes,
                              cudaStream_t st, const char **why) {
  (void)ws_bytes;
  const bool pair_heads = ((Hq / Hkv) % 2) == 0;  // two heads of one GQA group per CTA
  if (D != 128 && D != 64) {
    *why = "tensor-core prefill: head_dim 64 or 128";
    return cudaErrorInvalidValue;
  }
  int *err = reinterpret_cast<int *>(ws);
  // grouped keys are needed unless the window keeps every visible pair local
  const bool any_grouped = !plain && !(window > 0 && window <= w0);
  const bool pre = (flags & JL_FLAG_PREROTATE_K) != 0 && any_grouped;
  __nv_bfloat16 *kg = pre ? reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<char *>(ws) + 256) : nullptr;
  CUtensorMap mQ, mK, mV, mKg;
  if (!make_map(&mQ, q, T_total, Hq, D) || !make_map(&mK, k, Tk, Hkv, D) || !make_map(&mV, v, Tk, Hkv, D) ||
      !make_map(&mKg, pre ? (const void *)kg : k, Tk, Hkv, D)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  if (pre) {
    const long long n = (long long)Tk * (D / 16);
    tc::prerotate_k_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16 *)k, kg, D, cu_k, batch, Tk, Hkv, w_pre, inv);
    if ((e = cudaGetLastError()) != cudaSuccess) {
      *why = "pre-rotation launch";
      return e;
    }
  }
  e = !pair_heads   ? (D == 128 ? cudaFuncSetAttribute(tc::bifocal_prefill_kernel<128>,
                                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                          tc::Geo<128>::P1_SMEM_ALLOC)
                                  : cudaFuncSetAttribute(tc::bifocal_prefill_kernel<64>,
                                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                          tc::Geo<64>::P1_SMEM_ALLOC))
      : D == 128 ? cudaFuncSetAttribute(tc::bifocal_prefill2_kernel<128>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Geo<128>::SMEM_ALLOC)
                 : cudaFuncSetAttribute(tc::bifocal_prefill2_kernel<64>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Geo<64>::SMEM_ALLOC);
  if (e != cudaSuccess) {
    *why = "smem attribute";
    return e;
  }
  tc::Params p;
  p.cu = cu;
  p.cu_k = cu_k;
  p.batch = batch;
  p.T = T_total;
  p.Tk = Tk;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.w_pre = w_pre;
  p.w0 = w0;
  p.plain = plain;
  p.window = window;
  p.kg_pre = pre ? 1 : 0;
  p.out = (__nv_bfloat16 *)out;
  p.lse = lse;
  p.err = err;
  p.sl2 = 1.4426950408889634f / sqrtf((float)D);
  if (pair_heads) {
    dim3 grid((max_seqlen + tc::BM - 1) / tc::BM * (Hq / Hkv / 2), Hkv, batch);
    if (D == 128)
      tc::bifocal_prefill2_kernel<128><<<grid, tc::P2_THREADS, tc::Geo<128>::SMEM_ALLOC, st>>>(mQ, mK, mV, mKg, p,
                                                                                                 inv);
    else
      tc::bifocal_prefill2_kernel<64><<<grid, tc::P2_THREADS, tc::Geo<64>::SMEM_ALLOC, st>>>(mQ, mK, mV, mKg, p,
                                                                                               inv);
  } else {
    dim3 grid((max_seqlen + tc::BM - 1) / tc::BM, Hq, batch);
    if (D == 128)
      tc::bifocal_prefill_kernel<128><<<grid, tc::P1_THREADS, tc::Geo<128>::P1_SMEM_ALLOC, st>>>(mQ, mK, mV, mKg,
                                                                                                  p, inv);
    else
      tc::bifocal_prefill_kernel<64><<<grid, tc::P1_THREADS, tc::Geo<64>::P1_SMEM_ALLOC, st>>>(mQ, mK, mV, mKg, p,
                                                                                                inv);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) *why = "tensor-core prefill launch";
  return e;
}

}  // namespace jl

// Host copy of the prefill tile schedule, for tests: the visits of query tile
// qt of a sequence with L queries over Lk keys, five ints each (key tile,
// grouped, masked, lo, hi), at most cap visits; returns the visit count, or -1
// for arguments outside the kernels' range.
extern "C" int jl_debug_prefill_visits(int L, int Lk, int w0, int window, int G, int qt, int *out, int cap) {
  using namespace jl::tc;
  if (L <= 0 || Lk < L || w0 < 0 || window < 0 || G < 1 || qt < 0 || qt * BM >= L || out == nullptr) return -1;
  Tile t;
  t.L = L;
  t.qt = qt;
  t.i0 = qt * BM;
  t.i1 = L - 1 < t.i0 + BM - 1 ? L - 1 : t.i0 + BM - 1;
  t.Lk = Lk;
  t.off = Lk - L;
  t.W = window;
  t.G = G;
  t.bif = G > 1;
  const VisitPlan pl = make_plan(t, w0);
  for (int v = 0; v < pl.n_all && v < cap; ++v) {
    int kt;
    Visit vx;
    visit_at(t, pl, w0, v, kt, vx);
    out[5 * v + 0] = kt;
    out[5 * v + 1] = vx.grp;
    out[5 * v + 2] = vx.mask;
    out[5 * v + 3] = vx.lo;
    out[5 * v + 4] = vx.hi;
  }
  return pl.n_all;
}

namespace jl {
// Test hook: the limit of the bounded waits of this file's kernels.
cudaError_t set_wait_limit_prefill(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}
}  // namespace jl
