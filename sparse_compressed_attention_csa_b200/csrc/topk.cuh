// Step 2b: exact top-k ("keeps the top 1,024 entries"), ties to the lower
// index, output in ascending index order and padded with -1.
//
// Radix select on order-preserving uint32 keys, 8 bits per pass from the
// most significant digit: each pass histograms the digit of the keys that
// still match the chosen prefix and picks the digit holding the k-th
// largest key.  After four passes the prefix is the exact threshold key T
// and `remaining` is how many keys equal to T are kept (the lowest indices
// among them).  A final pass in index order compacts the selection with
// block prefix sums, which makes the output ascending.
//
// k_topk_rows: one CTA per query row (any n).  Rows with at most k visible
// entries write 0..n_vis-1 and padding without reading scores.
#pragma once
#include "common.cuh"

namespace csa {

struct RadixState {
  uint32_t prefix;
  int remaining;
};

// Warp 0 picks the digit of the k-th largest key from a 256-bin histogram.
// Every thread of the block must call it (it synchronises).
__device__ __forceinline__ void radix_pick_digit(const unsigned* hist, int shift,
                                                 RadixState* st) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int need = st->remaining;
    int local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) local += (int)hist[lane * 8 + i];
    // suffix sum over lanes: sum of lanes >= lane
    int suf = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += n;
    }
    int above = __shfl_down_sync(0xffffffffu, suf, 1);
    if (lane == 31) above = 0;
    if (suf >= need && above < need) {
      int cum = above;
      for (int bin = lane * 8 + 7; bin >= lane * 8; --bin) {
        if (cum + (int)hist[bin] >= need) {
          st->prefix |= (uint32_t)bin << shift;
          st->remaining = need - cum;
          break;
        }
        cum += (int)hist[bin];
      }
    }
  }
  __syncthreads();
}

template <int NT>
__global__ void __launch_bounds__(NT)
    k_topk_rows(const float* __restrict__ scores, const int* __restrict__ q_pos,
                const int* __restrict__ n_cmp, int Tq, int n_max, int k, int width, int stride,
                int* __restrict__ idx_out) {
  __shared__ unsigned hist[256];
  __shared__ RadixState st;
  __shared__ int scan_tmp[33];
  const int row = blockIdx.x;
  const int b = row / Tq;
  const int nv = min(n_visible(q_pos[row], n_cmp[b], width, stride), n_max);
  int* out = idx_out + (size_t)row * k;
  if (nv <= k) {
    for (int i = threadIdx.x; i < k; i += NT) out[i] = i < nv ? i : -1;
    return;
  }
  const float* s = scores + (size_t)row * n_max;
  if (threadIdx.x == 0) {
    st.prefix = 0u;
    st.remaining = k;
  }
  uint32_t mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = st.prefix;
    for (int j = threadIdx.x; j < nv; j += NT) {
      const uint32_t key = float_key(s[j]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    radix_pick_digit(hist, shift, &st);
    mask |= 255u << shift;
  }
  const uint32_t thr = st.prefix;
  const int take_eq = st.remaining;
  int written = 0, eq_seen = 0;
  for (int base = 0; base < nv; base += NT) {
    const int j = base + threadIdx.x;
    uint32_t key = 0u;
    if (j < nv) key = float_key(s[j]);
    const int gt = (j < nv && key > thr) ? 1 : 0;
    const int eq = (j < nv && key == thr) ? 1 : 0;
    int eq_tot;
    const int eq_rank = block_inclusive_scan(eq, scan_tmp, &eq_tot) - eq;
    const int sel = gt | (eq & (eq_seen + eq_rank < take_eq ? 1 : 0));
    int sel_tot;
    const int pos = block_inclusive_scan(sel, scan_tmp, &sel_tot) - sel;
    if (sel && written + pos < k) out[written + pos] = j;
    written += sel_tot;
    eq_seen += eq_tot;
    if (written >= k) break;
  }
}

}  // namespace csa
