// Step 1: gated pooling of token KV rows into compressed entries, plus the
// rotated raw rows ("Compressed Sparse Attention" row: 8 overlapping tokens
// at stride 4 with a per-channel softmax; "Heavily Compressed Attention"
// row: 128 tokens -> 1 entry; "Partial RoPE" row), for a whole sequence or
// for the tokens one decode step appends.
//
// HBM-streaming kernel: each thread owns 16 bytes of channels (8 bf16 or 4
// fp32), so every load and store is a 16-byte vector and the threads of a
// row cover it contiguously.  One launch, three kinds of CTA (256 threads):
//  * wide entries (HCA's 128 tokens): one CTA per entry, its taps split over
//    256 / (d / VEC) thread groups whose partial softmax states merge in
//    shared memory;
//  * narrow entries (CSA's 8 taps): 256 / (d / VEC) entries per CTA, a
//    thread runs all taps of its channels; a token row is read by
//    width / stride entries and the overlap hits L2;
//  * raw rows: four tokens per thread, their loads in flight together.
// Softmax over the taps is the online (running max) form in fp32.  RoPE
// frequencies come from a per-launch table; the angle is reduced in double
// precision (rope_cs_reduced).
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kCompressThreads = 256;
constexpr int kCompressWideMin = 32;    // entries at least this wide take a CTA each
constexpr int kCompressRawPer = 4;      // raw rows per thread
constexpr int kCompressMaxPairs = 512;  // RoPE pairs in the table (rope_dim <= 1024)

// Per sequence b, the launch writes entries j = n_entries(t_lo) + r for r in
// [0, e_slots) while j < n_entries(t_hi), and raw rows of tokens t = t_lo + u
// for u in [0, n_raw) while t < t_hi, where t_lo = t_old[b] (0 when NULL)
// and t_hi = t_new[b] (T when NULL).  Token t is row t - x_pos0[b] of x and g;
// entry j is row j of kv_cmp; token t's raw row is row t - raw_pos0[b] of
// kv_raw.  A sequence whose range breaks t_lo <= t_hi <= t_lo + max_new
// is skipped, a row that would read or write outside a buffer too; both are
// recorded as CSA_ERR_DEVICE_BOUNDS.  CTAs [0, wide_ctas) are the wide
// entries (wide_ctas = e_slots when width >= kCompressWideMin, else 0); the
// rest hold the row slots: narrow_slots entries (e_slots, or 0 when wide),
// then raw_slots = ceil(n_raw / kCompressRawPer) groups of raw rows.
struct CompressArgs {
  const void* x;
  const void* g;
  const int32_t* x_pos0;
  int L;  // token rows per sequence in x and g
  const int32_t* t_old;
  const int32_t* t_new;
  int T;
  int max_new;  // bound on t_hi - t_lo (checked)
  int d, width, stride, pos_offset;
  RopeSpec rope;
  int n_raw;  // raw rows per sequence the launch covers (0: none)
  int wide_ctas, narrow_slots, raw_slots;
  void* kv_cmp;
  int n_cap;
  void* kv_raw;
  const int32_t* raw_pos0;
  int raw_cap;
  double freq[kCompressMaxPairs];  // RoPE frequency of pair i
};

__device__ __forceinline__ int n_entries(int t, int width, int stride) {
  return t < width ? 0 : (t - width) / stride + 1;
}

// 16 bytes of channels as floats, and back (bf16: round to nearest even).
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load16(const float* p, float (&v)[4]) {
  const float4 u = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = u.x;
  v[1] = u.y;
  v[2] = u.z;
  v[3] = u.w;
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void store16(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// Rotate the pairs (c0 + 2k, c0 + 2k + 1) that fall in the RoPE dims.
template <int VEC>
__device__ __forceinline__ void rotate16(float (&v)[VEC], int c0, int rope0, const double* freq,
                                         long long pos) {
  if (c0 + VEC <= rope0) return;
#pragma unroll
  for (int k = 0; k < VEC / 2; ++k) {
    const int c = c0 + 2 * k;
    if (c >= rope0) {
      float cs, sn;
      rope_cs_reduced(pos, freq[(c - rope0) / 2], &cs, &sn);
      const float a = v[2 * k], b = v[2 * k + 1];
      v[2 * k] = a * cs - b * sn;
      v[2 * k + 1] = a * sn + b * cs;
    }
  }
}

// Online softmax state of VEC channels over some taps, in the log2 domain
// (m is the running maximum of g * log2(e)), and its update: one exp2 per
// tap and channel, e = 2^-|l - m| for the tap's scaled logit l; a tap above
// the maximum rescales the sums by e and enters with weight 1, any other
// enters with weight e.
template <int VEC>
struct PoolState {
  float m[VEC], s[VEC], acc[VEC];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      m[k] = -INFINITY;
      s[k] = 0.f;
      acc[k] = 0.f;
    }
  }
  __device__ __forceinline__ void add(const float (&gv)[VEC], const float (&xv)[VEC]) {
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      const float l = gv[k] * 1.4426950408889634f;
      const float dl = l - m[k];
      const float e = exp2f(-fabsf(dl));
      const bool up = dl > 0.f;
      s[k] = up ? fmaf(s[k], e, 1.f) : s[k] + e;
      acc[k] = up ? fmaf(acc[k], e, xv[k]) : fmaf(e, xv[k], acc[k]);
      m[k] = up ? l : m[k];
    }
  }
};

template <typename T>
__global__ void __launch_bounds__(kCompressThreads, 4) k_compress(CompressArgs a) {
  constexpr int VEC = 16 / (int)sizeof(T);
  constexpr int kSlots = kCompressThreads * VEC;  // wide CTA: G * d channel states
  __shared__ float sm_m[kSlots], sm_s[kSlots], sm_acc[kSlots];
  const int tpr = a.d / VEC;               // threads per row
  const int rpc = kCompressThreads / tpr;  // row slots (or tap groups) per CTA
  const int sub = (int)threadIdx.x / tpr;
  const int c0 = ((int)threadIdx.x % tpr) * VEC;
  const int b = blockIdx.y;
  const int t_lo = a.t_old ? a.t_old[b] : 0;
  const int t_hi = a.t_new ? a.t_new[b] : a.T;
  if (t_hi < t_lo || t_hi - t_lo > a.max_new) {  // the sequence's range breaks the rules
    if (blockIdx.x == 0 && threadIdx.x == 0) report_error(CSA_ERR_DEVICE_BOUNDS);
    return;
  }
  const int xp0 = a.x_pos0 ? a.x_pos0[b] : 0;
  const T* xb = static_cast<const T*>(a.x) + (size_t)b * a.L * a.d;
  const T* gb = static_cast<const T*>(a.g) + (size_t)b * a.L * a.d;
  const int rope0 = a.d - a.rope.rope_dim;
  const int e0 = n_entries(t_lo, a.width, a.stride), e1 = n_entries(t_hi, a.width, a.stride);

  if ((int)blockIdx.x < a.wide_ctas) {
    // ---- one wide entry; tap group `sub` runs taps sub, sub + G, ...
    const int j = e0 + (int)blockIdx.x;
    if (j >= e1) return;  // uniform over the CTA
    const long long row0 = (long long)a.stride * j - xp0;
    if (j >= a.n_cap || row0 < 0 || row0 + a.width > a.L) {
      if (threadIdx.x == 0) report_error(CSA_ERR_DEVICE_BOUNDS);
      return;
    }
    const int G = min(rpc, a.width);
    if (sub < G) {
      const T* xr = xb + (size_t)row0 * a.d + c0;
      const T* gr = gb + (size_t)row0 * a.d + c0;
      PoolState<VEC> st;
      st.init();
#pragma unroll 4
      for (int u = sub; u < a.width; u += G) {
        float gv[VEC], xv[VEC];
        load16(gr + (size_t)u * a.d, gv);
        load16(xr + (size_t)u * a.d, xv);
        st.add(gv, xv);
      }
#pragma unroll
      for (int k = 0; k < VEC; ++k) {
        sm_m[sub * a.d + c0 + k] = st.m[k];
        sm_s[sub * a.d + c0 + k] = st.s[k];
        sm_acc[sub * a.d + c0 + k] = st.acc[k];
      }
    }
    __syncthreads();
    // merge: m = max_g m_g, s = sum_g s_g 2^(m_g - m), acc likewise; thread
    // i takes channel pairs i, i + 256, ... (a RoPE pair stays in one thread)
    T* dst = static_cast<T*>(a.kv_cmp) + ((size_t)b * a.n_cap + j) * a.d;
    const long long pos = (long long)a.stride * j + a.pos_offset;
    for (int pr = threadIdx.x; pr < a.d / 2; pr += kCompressThreads) {
      float v[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 2 * pr + h;
        float m = -INFINITY;
        for (int g = 0; g < G; ++g) m = fmaxf(m, sm_m[g * a.d + c]);
        float sum = 0.f, acc = 0.f;
        for (int g = 0; g < G; ++g) {
          const float w = exp2f(sm_m[g * a.d + c] - m);
          sum += sm_s[g * a.d + c] * w;
          acc += sm_acc[g * a.d + c] * w;
        }
        v[h] = acc / sum;
      }
      if (2 * pr >= rope0) {
        float cs, sn;
        rope_cs_reduced(pos, a.freq[(2 * pr - rope0) / 2], &cs, &sn);
        const float x0 = v[0], x1 = v[1];
        v[0] = x0 * cs - x1 * sn;
        v[1] = x0 * sn + x1 * cs;
      }
      store2(dst + 2 * pr, v[0], v[1]);
    }
    return;
  }

  const int r = ((int)blockIdx.x - a.wide_ctas) * rpc + sub;  // row slot
  if (r < a.narrow_slots) {
    // ---- one narrow entry: all taps of this thread's channels
    const int j = e0 + r;
    if (j >= e1) return;
    const long long row0 = (long long)a.stride * j - xp0;
    if (j >= a.n_cap || row0 < 0 || row0 + a.width > a.L) {
      report_error(CSA_ERR_DEVICE_BOUNDS);
      return;
    }
    PoolState<VEC> st;
    st.init();
    const T* xr = xb + (size_t)row0 * a.d + c0;
    const T* gr = gb + (size_t)row0 * a.d + c0;
#pragma unroll 4
    for (int u = 0; u < a.width; ++u) {
      float gv[VEC], xv[VEC];
      load16(gr + (size_t)u * a.d, gv);
      load16(xr + (size_t)u * a.d, xv);
      st.add(gv, xv);
    }
    float v[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) v[k] = st.acc[k] / st.s[k];
    rotate16<VEC>(v, c0, rope0, a.freq, (long long)a.stride * j + a.pos_offset);
    store16(static_cast<T*>(a.kv_cmp) + ((size_t)b * a.n_cap + j) * a.d + c0, v);
  } else if (r < a.narrow_slots + a.raw_slots) {
    // ---- raw rows of tokens t0 .. t0 + 3, loads first
    const int t0 = t_lo + (r - a.narrow_slots) * kCompressRawPer;
    const int rp0 = a.raw_pos0 ? a.raw_pos0[b] : 0;
    float v[kCompressRawPer][VEC];
    bool ok[kCompressRawPer];
#pragma unroll
    for (int q = 0; q < kCompressRawPer; ++q) {
      const int t = t0 + q;
      const long long src = (long long)t - xp0, dst = (long long)t - rp0;
      ok[q] = t < t_hi && t - t_lo < a.n_raw;
      if (ok[q] && (src < 0 || src >= a.L || dst < 0 || dst >= a.raw_cap)) {
        report_error(CSA_ERR_DEVICE_BOUNDS);
        ok[q] = false;
      }
      if (ok[q]) load16(xb + (size_t)src * a.d + c0, v[q]);
    }
#pragma unroll
    for (int q = 0; q < kCompressRawPer; ++q) {
      if (!ok[q]) continue;
      const int t = t0 + q;
      rotate16<VEC>(v[q], c0, rope0, a.freq, t);
      store16(static_cast<T*>(a.kv_raw) + ((size_t)b * a.raw_cap + (t - rp0)) * a.d + c0, v[q]);
    }
  }
}

}  // namespace csa
