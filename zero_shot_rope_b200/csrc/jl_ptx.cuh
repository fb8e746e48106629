// PTX helpers shared by the sm_100a kernels: mbarriers, bounded waits and
// TMA tensor loads.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace jl {

__device__ __forceinline__ uint32_t su32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Named barrier over `nthreads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded waits.  The limit of an ordinary wait is this device variable (one
// copy per translation unit), 2 s unless a test shortens it through
// jl_debug_set_wait_limit; the drain waits below keep a fixed 2 s.
static __device__ unsigned long long g_wait_limit_ns = 2000000000ull;

// A translation unit whose kernels rebalance registers with setmaxnreg
// defines JL_WAITS_INLINE before including this file: ptxas cannot compile
// function calls inside such kernels, so the slow paths are inlined there.
#ifdef JL_WAITS_INLINE
#define JL_WAIT_SLOW __forceinline__
#else
#define JL_WAIT_SLOW __noinline__
#endif

// Bounded wait: false on timeout (records `code`) or when another role aborted.
// The first probe is inlined: most waits on the pipelines' critical paths find
// the phase already complete, and a call there costs more than the probe.
static __device__ JL_WAIT_SLOW bool wait_b_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                int *gerr, int code) {
  const uint64_t t0 = gtime();
  const uint64_t limit = *(volatile unsigned long long *)&g_wait_limit_ns;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (gtime() - t0 > limit) {
        *abort_flag = 1;
        if (gerr) atomicOr(gerr, code);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_b(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *gerr,
                                       int code) {
  if (mbar_try(bar, parity)) return true;
  return wait_b_slow(bar, parity, abort_flag, gerr, code);
}
// Bounded wait used only to let this CTA's own copies / MMAs land before it
// exits; ignores the abort flag and keeps a fixed limit.
static __device__ JL_WAIT_SLOW void wait_drain(uint64_t *bar, uint32_t parity, int *gerr, int code) {
  const uint64_t t0 = gtime();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try(bar, parity)) return;
    if ((it & 31u) == 31u && gtime() - t0 > 2000000000ull) {
      atomicOr(gerr, code);
      return;
    }
  }
}
__device__ __forceinline__ void tma_load(const CUtensorMap *map, uint64_t *bar, uint32_t dst, int c0,
                                         int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(su32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// The same load with an L2 eviction-priority policy (from createpolicy).
__device__ __forceinline__ void tma_load_hint(const CUtensorMap *map, uint64_t *bar, uint32_t dst, int c0, int c1,
                                              int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(map), "r"(su32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
// L2 policies: keep lines that other CTAs will read again; let once-read lines go first.
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte global store with an L2 eviction-priority policy.
__device__ __forceinline__ void stg128_hint(void *p, uint4 x, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(x.x), "r"(x.y), "r"(x.z),
               "r"(x.w), "l"(policy)
               : "memory");
}

__device__ __forceinline__ float ex2(float x) {  // MUFU exp2 (ex2.approx.ftz)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Host: cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace jl
