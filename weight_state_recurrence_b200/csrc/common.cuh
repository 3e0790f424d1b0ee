// Element types, the feature map and small helpers shared by the kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace linattn {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Eight consecutive elements as fp32, from an address aligned to eight
// elements (one 16-byte load for bf16, two for fp32).
template <typename T>
__device__ __forceinline__ void load8_f32(const T *p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8_f32<float>(const float *p, float (&f)[8]) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0];
  const float4 b = reinterpret_cast<const float4 *>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
template <>
__device__ __forceinline__ void load8_f32<__nv_bfloat16>(const __nv_bfloat16 *p, float (&f)[8]) {
  const uint4 w = *reinterpret_cast<const uint4 *>(p);
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(ww[i] << 16);
    f[2 * i + 1] = __uint_as_float(ww[i] & 0xffff0000u);
  }
}

// phi(x) = elu(x) + 1 (alpha = 1): x + 1 for x > 0, exp(x) otherwise.
// Fast-weight article §4.1 (feature_map); linear-attention note §4.1.
__device__ __forceinline__ float phi_f32(float x) { return x > 0.f ? x + 1.f : expf(x); }

// The feature applied to a q or k element: elu + 1, or none (`ident`) when q
// and k already hold feature vectors, such as random features computed
// beforehand.
__device__ __forceinline__ float feat_f32(float x, bool ident) { return ident ? x : phi_f32(x); }

// lambda^i for integer i >= 0 by binary exponentiation in fp32 (at most
// 2*log2(i) roundings).  lambda^0 = 1 also for lambda = 0.  Powers are
// always formed directly, never as a ratio lambda^a / lambda^b, which would
// overflow for small lambda.
__device__ __forceinline__ float pow_int(float L, int i) {
  float r = 1.f, b = L;
  while (i > 0) {
    if (i & 1) r *= b;
    b *= b;
    i >>= 1;
  }
  return r;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace linattn
