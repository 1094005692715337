// Step 2a, generic shapes: lightning-indexer scores on CUDA cores
// ("Compressed Sparse Attention" row: 64 heads x 128 dims, ReLU scores
// weighted per head).  s[t][j] = sum_h w[t][h] * max(0, q[t][h] . k[j]).
//
// One CTA per (sequence, query token, 128 keys); the query's indexer heads
// and weights sit in shared memory, each thread scores one key with fp32
// FMAs, 16 heads at a time.  The tensor-core kernel in indexer_tc.cuh
// replaces this one for the measured shape (64 x 128, bf16).
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kIdxSimtKeys = 128;

template <typename T>
__global__ void __launch_bounds__(kIdxSimtKeys)
    k_index_scores_simt(const T* __restrict__ q_idx, const float* __restrict__ w,
                        const T* __restrict__ k_idx, const int* __restrict__ q_pos,
                        const int* __restrict__ n_cmp, int Tq, int n_max, int H_I, int d_I,
                        int width, int stride, float* __restrict__ scores) {
  extern __shared__ float smem[];
  float* qs = smem;               // [H_I][d_I]
  float* ws = smem + H_I * d_I;   // [H_I]
  const int b = blockIdx.z, t = blockIdx.y;
  const int row = b * Tq + t;
  // counts from device memory are clamped to the buffer (n_cmp <= n_max)
  const int nv = min(n_visible(q_pos[row], n_cmp[b], width, stride), n_max);
  const int j0 = blockIdx.x * kIdxSimtKeys;
  if (j0 >= nv) return;
  const T* qrow = q_idx + (size_t)row * H_I * d_I;
  for (int i = threadIdx.x; i < H_I * d_I; i += blockDim.x) qs[i] = to_f32(qrow[i]);
  for (int i = threadIdx.x; i < H_I; i += blockDim.x) ws[i] = w[(size_t)row * H_I + i];
  __syncthreads();
  const int j = j0 + threadIdx.x;
  if (j >= nv) return;
  const T* key = k_idx + ((size_t)b * n_max + j) * d_I;
  float score = 0.f;
  for (int h0 = 0; h0 < H_I; h0 += 16) {
    const int nh = min(16, H_I - h0);
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    for (int c = 0; c < d_I; c += 2) {
      const float2 kv = load2(key + c);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < nh) {
          acc[i] = fmaf(qs[(h0 + i) * d_I + c], kv.x, acc[i]);
          acc[i] = fmaf(qs[(h0 + i) * d_I + c + 1], kv.y, acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < nh) score = fmaf(ws[h0 + i], fmaxf(acc[i], 0.f), score);
  }
  scores[(size_t)row * n_max + j] = score;
}

}  // namespace csa
