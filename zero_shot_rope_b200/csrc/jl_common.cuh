// Shared device helpers of the Dynamic Bifocal RoPE kernels.
//
// Position policy (Jet-Long technical summary, §1 "RoPE Bifocal Dinâmico"):
//   G = max(1, ceil(L / w_pretrained)),  f(x) = floor(x / G),
// and the correction shift of §2 "Rotação de Correção On-the-Fly":
//   delta(p) = f(p) - p  (<= 0), so R(delta(p)) R(p) = R(f(p)).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define JL_MAX_HALF 64  // D/2 for the largest supported head_dim (128)

namespace jl {

// fp64 RoPE inverse frequencies theta^(-2k/D), computed on the host once per
// call and passed by value.
struct InvFreq {
  double v[JL_MAX_HALF];
};

__host__ __device__ __forceinline__ int64_t group_size(int64_t L, int64_t w) {
  int64_t g = (L + w - 1) / w;
  return g < 1 ? 1 : g;
}

// floor(x / G) for x >= 0.
__host__ __device__ __forceinline__ int32_t fmap(int32_t x, int32_t G) { return x / G; }

// n(p) = p - f(p) >= 0: the correction rotates by -n(p) positions.
__host__ __device__ __forceinline__ int32_t corr_n(int32_t p, int32_t G) { return p - p / G; }

// sin and cos of an fp64 angle x, |x| < 2^40, with no function call (so it
// may run inside kernels that rebalance registers with setmaxnreg, where
// ptxas cannot handle calls).  Cody–Waite reduction by pi/2: k = rint(x 2/pi)
// and r = x - k pi/2 in two fused multiply-adds against pi/2 written as the
// sum of two doubles, exact to ~1e-16 for every k < 2^53; then the Taylor
// series of sin (to r^17) and cos (to r^16) on |r| <= pi/4, whose truncation
// errors are below 1e-19; then the quadrant k mod 4.
__host__ __device__ __forceinline__ void sincos_fp64(double x, double &sn, double &cs) {
  const double two_over_pi = 0.63661977236758134308;
  const double pio2_hi = 1.5707963267948966192;     // fp64 nearest to pi/2
  const double pio2_lo = 6.1232339957367660359e-17;  // pi/2 - pio2_hi
  const double k = rint(x * two_over_pi);
  double r = fma(-k, pio2_hi, x);
  r = fma(-k, pio2_lo, r);
  const double r2 = r * r;
  double ps = 1.0 / 355687428096000.0;  // 1/17!
  ps = fma(ps, -r2, 1.0 / 1307674368000.0);
  ps = fma(ps, -r2, 1.0 / 6227020800.0);
  ps = fma(ps, -r2, 1.0 / 39916800.0);
  ps = fma(ps, -r2, 1.0 / 362880.0);
  ps = fma(ps, -r2, 1.0 / 5040.0);
  ps = fma(ps, -r2, 1.0 / 120.0);
  ps = fma(ps, -r2, 1.0 / 6.0);
  const double sr = fma(-r * r2, ps, r);  // r - r^3/3! + r^5/5! - ...
  double pc = 1.0 / 20922789888000.0;   // 1/16!
  pc = fma(pc, -r2, 1.0 / 87178291200.0);
  pc = fma(pc, -r2, 1.0 / 479001600.0);
  pc = fma(pc, -r2, 1.0 / 3628800.0);
  pc = fma(pc, -r2, 1.0 / 40320.0);
  pc = fma(pc, -r2, 1.0 / 720.0);
  pc = fma(pc, -r2, 1.0 / 24.0);
  pc = fma(pc, -r2, 1.0 / 2.0);
  const double cr = fma(-r2, pc, 1.0);  // 1 - r^2/2! + r^4/4! - ...
  switch ((long long)k & 3) {
    case 0: sn = sr; cs = cr; break;
    case 1: sn = cr; cs = -sr; break;
    case 2: sn = -sr; cs = -cr; break;
    default: sn = -cr; cs = sr; break;
  }
}

// cos / sin of the angle n * invf, formed in fp64 from the exact integer n and
// evaluated in fp64 before rounding to fp32.
__host__ __device__ __forceinline__ void angle_cs(int32_t n, double invf, float &c, float &s) {
  double sd, cd;
  sincos_fp64((double)n * invf, sd, cd);
  c = (float)cd;
  s = (float)sd;
}

// Rotate the pair (a, b) by -n positions given c = cos(n w), s = sin(n w):
//   R(-n)(a, b) = (a c + b s, -a s + b c).
__device__ __forceinline__ void rot_back(float &a, float &b, float c, float s) {
  float a2 = fmaf(a, c, b * s);
  float b2 = fmaf(b, c, -(a * s));
  a = a2;
  b = b2;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace jl
