// Step 1: gated pooling of token KV rows into compressed entries, plus the
// rotated raw rows ("Compressed Sparse Attention" row: 8 overlapping tokens
// at stride 4 with a per-channel softmax; "Heavily Compressed Attention"
// row: 128 tokens -> 1 entry; "Partial RoPE" row).
//
// HBM-streaming kernel: one CTA per output row (pooled entry or raw row) of
// one sequence, one thread per channel pair (2c, 2c+1) so that the RoPE pair
// of a rotated channel lives in one thread.  Each token row is read by
// width/stride entries; the overlap hits L2.  Softmax over the taps is the
// online (running max) form in fp32.
#pragma once
#include "common.cuh"

namespace csa {

template <typename T>
__global__ void __launch_bounds__(256) k_compress(const T* __restrict__ x, const T* __restrict__ g,
                                                  int T_len, int d, int N, int width, int stride,
                                                  RopeSpec rope, int pos_offset,
                                                  T* __restrict__ kv_cmp, T* __restrict__ kv_raw) {
  const int b = blockIdx.y;
  const int r = blockIdx.x;
  const T* xb = x + (size_t)b * T_len * d;
  const T* gb = g + (size_t)b * T_len * d;
  const int rope0 = d - rope.rope_dim;
  if (r < N) {
    const long long pos = (long long)stride * r + pos_offset;
    T* dst = kv_cmp + ((size_t)b * N + r) * d;
    for (int c2 = threadIdx.x; c2 < d / 2; c2 += blockDim.x) {
      const int c = 2 * c2;
      float m0 = -INFINITY, m1 = -INFINITY, s0 = 0.f, s1 = 0.f, a0 = 0.f, a1 = 0.f;
      for (int u = 0; u < width; ++u) {
        const size_t off = (size_t)(stride * r + u) * d + c;
        const float2 gv = load2(gb + off);
        const float2 xv = load2(xb + off);
        const float n0 = fmaxf(m0, gv.x), n1 = fmaxf(m1, gv.y);
        const float r0 = expf(m0 - n0), r1 = expf(m1 - n1);
        const float e0 = expf(gv.x - n0), e1 = expf(gv.y - n1);
        s0 = s0 * r0 + e0;
        s1 = s1 * r1 + e1;
        a0 = a0 * r0 + e0 * xv.x;
        a1 = a1 * r1 + e1 * xv.y;
        m0 = n0;
        m1 = n1;
      }
      float v0 = a0 / s0, v1 = a1 / s1;
      if (c >= rope0) {
        float cs, sn;
        rope_cos_sin(pos, rope_freq(rope, (c - rope0) / 2), &cs, &sn);
        const float w0 = v0 * cs - v1 * sn, w1 = v0 * sn + v1 * cs;
        v0 = w0;
        v1 = w1;
      }
      store2(dst + c, v0, v1);
    }
  } else {
    const int t = r - N;
    const T* src = xb + (size_t)t * d;
    T* dst = kv_raw + ((size_t)b * T_len + t) * d;
    for (int c2 = threadIdx.x; c2 < d / 2; c2 += blockDim.x) {
      const int c = 2 * c2;
      float2 v = load2(src + c);
      if (c >= rope0) {
        float cs, sn;
        rope_cos_sin(t, rope_freq(rope, (c - rope0) / 2), &cs, &sn);
        v = make_float2(v.x * cs - v.y * sn, v.x * sn + v.y * cs);
      }
      store2(dst + c, v.x, v.y);
    }
  }
}

}  // namespace csa
