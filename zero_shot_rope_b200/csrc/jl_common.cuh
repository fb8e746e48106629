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

// cos / sin of the angle n * invf, formed in fp64 from the exact integer n and
// evaluated with the fp64 sincos before rounding to fp32.
__device__ __forceinline__ void angle_cs(int32_t n, double invf, float &c, float &s) {
  double sd, cd;
  sincos((double)n * invf, &sd, &cd);
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
