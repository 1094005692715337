// Shared device helpers of the CSA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// Per-device error word: kernels record the first device-side failure here
// (a bounded wait that ran out, a failed index check), and beside it the
// source line of the check that recorded it; csa_poll_device_error reads and
// clears both.  Never trap: the context stays usable.
__device__ int g_device_error;
__device__ int g_device_error_site;

__device__ __forceinline__ void report_error(int code, int site = __builtin_LINE()) {
  if (atomicCAS(&g_device_error, 0, code) == 0) atomicExch(&g_device_error_site, site);
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store(float* p, float v) { *p = v; }
__device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Load two consecutive elements (c, c+1) as floats.
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ void store2(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
__device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}

// RoPE ("Partial RoPE" row: rotate the trailing rope_dim of d dims).  Pair
// i is dims (d - rope_dim + 2i, d - rope_dim + 2i + 1), angle pos * f_i.
// f_i = theta^(-2i/rope_dim), or, for the compressed layers' extended RoPE
// (same row: theta 160,000 with YaRN, factor 16 over 65,536 tokens), the
// YaRN frequency of the published definition (Peng et al. 2023, section 3):
// a pair that turns n_i = L f_i / (2 pi) times over the original context L
// gets (1 - g) f_i / s + g f_i with g = clamp((n_i - alpha) / (beta - alpha),
// 0, 1).
struct RopeSpec {
  int rope_dim;
  double theta;
  double factor;    // s; <= 1: plain RoPE
  double orig_ctx;  // L
  double beta_fast; // beta
  double beta_slow; // alpha
};

__host__ __device__ inline double rope_freq(const RopeSpec& r, int i) {
  double f = pow(r.theta, -2.0 * (double)i / (double)r.rope_dim);
  if (r.factor > 1.0) {
    const double turns = r.orig_ctx * f / 6.283185307179586;
    double g = (turns - r.beta_slow) / (r.beta_fast - r.beta_slow);
    g = g < 0.0 ? 0.0 : (g > 1.0 ? 1.0 : g);
    f = (1.0 - g) * f / r.factor + g * f;
  }
  return f;
}

// cos / sin of pos * freq, the angle and its sine and cosine taken in double
// precision so that positions up to 2^20 keep full fp32 accuracy.
__device__ __forceinline__ void rope_cos_sin(long long pos, double freq, float* c, float* s) {
  double sd, cd;
  sincos((double)pos * freq, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

// cos / sin of pos * freq for the tensor-core and streaming kernels: the
// angle is formed in double precision and reduced modulo 2 pi there (2 pi
// split into a double and its remainder, a Cody-Waite reduction), and the
// reduced angle, in [-pi, pi], goes to the hardware sine / cosine (absolute
// error about 5e-7 on that range).  The angle's own error stays near 1e-16
// of pos * freq, so positions up to 2^20 lose nothing more.
__device__ __forceinline__ void rope_cs_reduced(long long pos, double freq, float* c, float* s) {
  const double x = (double)pos * freq;
  const double k = rint(x * 0.15915494309189535);
  double r = fma(-k, 6.283185307179586, x);
  r = fma(-k, 2.4492935982947064e-16, r);
  __sincosf((float)r, s, c);
}

// Entries j < n_cmp whose last pooled token s*j + w - 1 is at most t.
__device__ __forceinline__ int n_visible(int t, int n_cmp, int width, int stride) {
  if (t < width - 1) return 0;
  int v = (t - width + 1) / stride + 1;
  return v < n_cmp ? v : n_cmp;
}

// Order-preserving map fp32 -> uint32 (larger float, larger key); -0.0 is
// folded onto +0.0 so the two tie.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive block-wide prefix sum of one int per thread (blockDim.x a
// multiple of 32, at most 1024).  `tmp` holds >= 33 ints of shared memory.
// Returns the inclusive sum; *total receives the block total.
__device__ __forceinline__ int block_inclusive_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) tmp[wid] = v;
  __syncthreads();
  if (wid == 0) {
    int w = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < nw) tmp[lane] = w;  // inclusive warp totals
    if (lane == 31) tmp[32] = w;
  }
  __syncthreads();
  if (wid > 0) v += tmp[wid - 1];
  *total = tmp[32];
  __syncthreads();
  return v;
}

}  // namespace csa
