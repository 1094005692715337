// KV cache quantized after RoPE ("DeepSeek-V4.1-Flash vs Inkling", "Partial
// RoPE" row; the pages give no format): OCP E4M3 codes with one fp32 scale
// per row, scale = max|row| / 448 (1 for an all-zero row), code = x / scale
// rounded to the nearest E4M3 value (ties to even), saturated at +-448.  The
// scale and the division are IEEE fp32 (correctly rounded), the conversion
// the hardware's round-to-nearest with saturation.
//
// One warp per row; each lane takes groups of 8 channels (16-byte loads of
// bf16, 8-byte stores of codes), a warp max for the scale, then the codes.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa {

constexpr int kQuantWarps = 8;

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(32 * kQuantWarps)
    k_quantize_fp8(const T* __restrict__ rows, long long n, int d, uint8_t* __restrict__ codes,
                   float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (row >= n) return;
  const T* src = rows + row * d;
  float amax = 0.f;
  for (int c = 8 * lane; c < d; c += 256) {
    float v[8];
    load8(src + c, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[k]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* dst = codes + row * d;
  for (int c = 8 * lane; c < d; c += 256) {
    float v[8];
    load8(src + c, v);
    uint32_t w[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(v[4 * k], scale), __fdiv_rn(v[4 * k + 1], scale)), __NV_SATFINITE,
          __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(v[4 * k + 2], scale), __fdiv_rn(v[4 * k + 3], scale)),
          __NV_SATFINITE, __NV_E4M3);
      w[k] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    *reinterpret_cast<uint2*>(dst + c) = make_uint2(w[0], w[1]);
  }
  if (lane == 0) scales[row] = scale;
}

}  // namespace csa
