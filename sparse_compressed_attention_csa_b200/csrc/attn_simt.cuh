// Steps 3 and 4, generic shapes: shared-KV MQA over the selected compressed
// entries (CSA) or every visible entry (HCA), plus the raw window, with the
// per-head sink in the denominator and partial RoPE on q and on the output
// ("Compressed Sparse Attention", "Heavily Compressed Attention",
// "Partial RoPE" and "Output gate + sink" rows).
//
// CUDA-core kernel, fp32 math: one CTA of 4 warps per (sequence, query
// token, head).  Each warp runs an online softmax over every 4th row; lane l
// holds dims l, l+32, ...; the four partial states are merged with the sink
// at the end.  This is the path for fp32 and for shapes the tensor-core
// kernel does not cover.
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kAttnSimtWarps = 4;

struct AttnArgs {
  const void* q;
  const int* q_pos;
  const void* kv_cmp;
  const int* idx;    // CSA: [B][Tq][topk]
  const int* n_cmp;  // HCA: [B]
  int n_max;
  const void* kv_raw;
  const int* raw_pos0;
  const int* n_raw;
  int raw_max;
  const float* sink;
  const float* cmp_scale;  // FP8 caches (tensor-core path only): row scales
  const float* raw_scale;
  int layers;  // tensor-core path: layers sharing entries and selection (q, sink, out per layer)
  int B, Tq, H, d, rope_dim, topk, window, width, stride;
  float scale;  // with the extended RoPE's temperature
  RopeSpec rope;
  void* out;
};

// Rotate the lane's values (dims c = lane + 32*k) at position pos: pairs
// (2i, 2i+1) of the rope range sit in neighbouring lanes.
template <int NK>
__device__ __forceinline__ void rotate_lane_dims(float* v, int d, const RopeSpec& rope,
                                                 long long pos) {
  const int lane = threadIdx.x & 31;
  const int rope0 = d - rope.rope_dim;
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const int c = lane + 32 * k;
    const bool active = c >= rope0;  // uniform per k for rope0 % 32 == 0
    const float other = __shfl_xor_sync(0xffffffffu, v[k], 1);
    if (active) {
      float cs, sn;
      rope_cos_sin(pos, rope_freq(rope, (c - rope0) >> 1), &cs, &sn);
      v[k] = (c & 1) ? (other * sn + v[k] * cs) : (v[k] * cs - other * sn);
    }
  }
}

// NK = d / 32 values per lane.
template <typename T, bool kHca, int NK>
__global__ void __launch_bounds__(32 * kAttnSimtWarps) k_attn_simt(AttnArgs a) {
  __shared__ float sm_acc[kAttnSimtWarps][1024];
  __shared__ float sm_m[kAttnSimtWarps], sm_l[kAttnSimtWarps];
  const int h = blockIdx.x, tq = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int d = a.d;
  const int row = b * a.Tq + tq;
  const int t = a.q_pos[row];

  float qv[NK];
  const T* qp = reinterpret_cast<const T*>(a.q) + ((size_t)row * a.H + h) * d;
  _Pragma("unroll") for (int k = 0; k < NK; ++k) qv[k] = to_f32(qp[lane + 32 * k]);
  rotate_lane_dims<NK>(qv, d, a.rope, t);

  // rows: n_sel compressed entries, then the window's raw rows
  int n_sel;
  const int* sel = nullptr;
  if (kHca) {
    n_sel = min(n_visible(t, a.n_cmp[b], a.width, a.stride), a.n_max);
  } else {
    n_sel = a.topk;
    sel = a.idx + (size_t)row * a.topk;
  }
  const int rp0 = a.raw_pos0[b];
  int w_lo = max(max(0, t - a.window + 1), rp0);
  int w_hi = min(t, rp0 + min(a.n_raw[b], a.raw_max) - 1);
  const int n_win = a.window > 0 && w_hi >= w_lo ? w_hi - w_lo + 1 : 0;
  const int n_rows = n_sel + n_win;

  float m = -INFINITY, l = 0.f;
  float acc[NK];
  _Pragma("unroll") for (int k = 0; k < NK; ++k) acc[k] = 0.f;
  const T* cmp = reinterpret_cast<const T*>(a.kv_cmp) + (size_t)b * a.n_max * d;
  const T* raw = reinterpret_cast<const T*>(a.kv_raw) + (size_t)b * a.raw_max * d;
  for (int r = wid; r < n_rows; r += kAttnSimtWarps) {
    const T* src;
    if (r < n_sel) {
      int j = kHca ? r : sel[r];
      if (j < 0) continue;
      if (j >= a.n_max) {
        if (lane == 0) report_error(CSA_ERR_DEVICE_BOUNDS);
        continue;
      }
      src = cmp + (size_t)j * d;
    } else {
      src = raw + (size_t)(w_lo + (r - n_sel) - rp0) * d;
    }
    float rv[NK];
    float dot = 0.f;
    _Pragma("unroll") for (int k = 0; k < NK; ++k) {
      rv[k] = to_f32(src[lane + 32 * k]);
      dot = fmaf(qv[k], rv[k], dot);
    }
    const float z = warp_sum(dot) * a.scale;
    const float mn = fmaxf(m, z);
    const float alpha = expf(m - mn), p = expf(z - mn);
    l = l * alpha + p;
    _Pragma("unroll") for (int k = 0; k < NK; ++k) acc[k] = fmaf(p, rv[k], acc[k] * alpha);
    m = mn;
  }
  _Pragma("unroll") for (int k = 0; k < NK; ++k) sm_acc[wid][lane + 32 * k] = acc[k];
  if (lane == 0) {
    sm_m[wid] = m;
    sm_l[wid] = l;
  }
  __syncthreads();
  if (wid != 0) return;
  const float sink = a.sink[h];
  float M = sink;
  for (int w = 0; w < kAttnSimtWarps; ++w) M = fmaxf(M, sm_m[w]);
  // M == -inf only with a -inf sink and no rows: the output is 0.
  float scl[kAttnSimtWarps];
  float L = M == -INFINITY ? 1.f : expf(sink - M);
  for (int w = 0; w < kAttnSimtWarps; ++w) {
    scl[w] = sm_m[w] == -INFINITY ? 0.f : expf(sm_m[w] - M);
    L += sm_l[w] * scl[w];
  }
  const float inv = M == -INFINITY ? 0.f : 1.f / L;
  float o[NK];
  _Pragma("unroll") for (int k = 0; k < NK; ++k) {
    float s = 0.f;
    for (int w = 0; w < kAttnSimtWarps; ++w) s = fmaf(sm_acc[w][lane + 32 * k], scl[w], s);
    o[k] = s * inv;
  }
  rotate_lane_dims<NK>(o, d, a.rope, -(long long)t);
  T* op = reinterpret_cast<T*>(a.out) + ((size_t)row * a.H + h) * d;
  _Pragma("unroll") for (int k = 0; k < NK; ++k) store(op + lane + 32 * k, o[k]);
}

}  // namespace csa
