// Steps 3 and 4 on tensor cores, for the measured shape (128 query heads x
// 512 dims, bf16): shared-KV MQA over the selected compressed entries (CSA)
// or every visible entry (HCA), plus the raw window, with the per-head sink
// and partial RoPE ("Compressed Sparse Attention", "Heavily Compressed
// Attention", "Partial RoPE" and "Output gate + sink" rows).
//
// One query token = one MMA M of 128 heads.  Its output O (128 x 512 fp32)
// alone would fill all of TMEM (128 lanes x 512 columns), so every unit of
// work is split in two CTAs by output dims: CTA `half` owns d_v columns
// [256*half, 256*half + 256) and recomputes S = Q K^T itself.  Per CTA:
//
//   TMEM  O_half [0,256) | S0 [256,320) | S1 [320,384) | Q_other [384,512)
//   SMEM  Q_own (64 KB) | ring of 9 key/value chunks (16 KB each) | row list
//
// Q (rotated at the query position, rounded to bf16) is split by dims: the
// CTA's own 256 dims sit in shared memory (SS MMAs), the other 256 in TMEM
// (TS MMAs).  KV rows are gathered 64 at a time; each row is streamed as four
// 128-dim chunks (16 B cp.async, 128B-swizzled).  The two chunks of the
// other half feed only S and are released right after; the own two feed S
// and then, as V, the PV product, and are held until it completes.
//
//   warp 8 (one thread): MMAs   S(i) = Q K_i^T  (N = 64, K = 512)
//                               O   += P(i-1) V(i-1)  (A = P from TMEM, N = 2 x 128)
//   warps 4-7: gather producers (cp.async, zero-filled tails)
//   warps 0-3: one head per thread (= TMEM lane): online softmax in the
//              log2 domain with a lazy rescale (only when the running max
//              grows by more than 2^8), P written back over S as bf16,
//              epilogue with the sink, the inverse output rotation and the
//              store (or split-KV partials).
// Every mbarrier wait is bounded; a timeout records CSA_ERR_DEVICE_TIMEOUT
// and the CTA winds down, frees TMEM and exits.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kAtHeads = 128;
constexpr int kAtDim = 512;
constexpr int kAtTile = 64;          // KV rows per S tile (MMA N)
constexpr int kAtChunkBytes = kAtTile * 128 * 2;  // 64 rows x 128 dims bf16
constexpr int kAtR1 = 3;             // ring of "other half" chunks
constexpr int kAtR2 = 6;             // ring of "own half" chunks (V)
constexpr int kAtRowCap = 2048;      // rows per query token (selected + window)
constexpr int kAtThreads = 288;
constexpr float kAtRescaleLog2 = 8.0f;

struct AtSmem {
  alignas(1024) uint8_t q_own[4][kAtHeads * 128];          // 4 x [128 heads][64 dims]
  alignas(1024) uint8_t r1[kAtR1][kAtChunkBytes];          // [2][64 rows][128 B]
  alignas(1024) uint8_t r2[kAtR2][kAtChunkBytes];
  int rows[kAtRowCap];
  const __nv_bfloat16* row_ptr[2][kAtTile];                // per tile parity
  float cs[256], sn[256];
  uint64_t r1_full[kAtR1], r1_empty[kAtR1], r2_full[kAtR2], r2_empty[kAtR2];
  uint64_t s_full[2], p_full[2], pv_done[2], q_tma, q_ready, rows_ready;
  uint32_t tmem_base;
  int n_rows;
  int abort_flag;
  int prod_ok;
};

struct AttnTcArgs {
  const __nv_bfloat16* q;
  const int* q_pos;
  const __nv_bfloat16* kv_cmp;
  const int* idx;    // CSA
  const int* n_cmp;  // HCA
  int n_max;
  const __nv_bfloat16* kv_raw;
  const int* raw_pos0;
  const int* n_raw;
  int raw_max;
  const float* sink;
  int Tq, topk, window, width, stride, rope_dim;
  float scale_log2;
  double theta;
  int splits;
  __nv_bfloat16* out;  // splits == 1
  float* part_o;       // splits > 1: [B*Tq][splits][2][128][256]
  float* part_ml;      // [B*Tq][splits][2][2][128]  (m, l)
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Arrive (without changing the expected count) on `bar` once every cp.async
// this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                   sm100::smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of 16-byte unit u (0..7) of row r inside a 128B-swizzled
// [rows][128 B] block (atoms of 8 rows).
__device__ __forceinline__ uint32_t swz(int r, int u) {
  return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
}

template <bool kHca>
__global__ void __launch_bounds__(kAtThreads, 1)
    k_attn_tc(AttnTcArgs a, const __grid_constant__ CUtensorMap tm_q) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  AtSmem& sm = *reinterpret_cast<AtSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
  const int half = blockIdx.x & 1;
  const int split = blockIdx.x >> 1;
  const int row_q = blockIdx.y;  // b * Tq + tq
  const int b = row_q / a.Tq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = a.q_pos[row_q];
  const int rope0 = kAtDim - a.rope_dim;
  const int own0 = 2 * half;  // own 128-dim chunks: own0, own0 + 1 (dims 256*half ..)
  const int oth0 = 2 * (1 - half);
  // staging of the other half of q (4 sub-blocks of [128 heads][64 dims])
  uint8_t* q_stage = sm.r2[kAtR2 - 4];

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAtR1; ++s) {
      mbar_init(&sm.r1_full[s], 128);
      mbar_init(&sm.r1_empty[s], 1);
    }
    for (int s = 0; s < kAtR2; ++s) {
      mbar_init(&sm.r2_full[s], 128);
      mbar_init(&sm.r2_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.pv_done[i], 1);
    }
    mbar_init(&sm.q_tma, 1);
    mbar_init(&sm.q_ready, 128);
    mbar_init(&sm.rows_ready, 128);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t t_o = tmem, t_s = tmem + 256, t_q = tmem + 384;
  volatile int* abortp = &sm.abort_flag;

  if (warp == 4 && lane == 0) {
    // q of this token: 8 boxes of [128 heads][64 dims] (128B swizzle); own
    // half straight to its place, other half to the staging slots
    tma_prefetch_desc(&tm_q);
    mbar_arrive_expect_tx(&sm.q_tma, kAtHeads * kAtDim * 2);
    for (int sb = 0; sb < 8; ++sb) {
      const bool own = (sb >> 2) == half;
      uint8_t* dst = own ? sm.q_own[sb & 3] : q_stage + (sb & 3) * (kAtHeads * 128);
      tma_load_2d(dst, &tm_q, &sm.q_tma, sb * 64, row_q * kAtHeads);
    }
  }

  if (warp < 4) {
    // ======================= softmax / epilogue warps
    // ---- RoPE table at the query position
    if (threadIdx.x < a.rope_dim / 2) {
      float c, s;
      rope_cos_sin(t, threadIdx.x, a.rope_dim, a.theta, &c, &s);
      sm.cs[threadIdx.x] = c;
      sm.sn[threadIdx.x] = s;
    }
    // ---- row list: selected (or visible) entries, then the window's raw rows
    int base = 0;
    if (kHca) {
      const int nv = min(n_visible(t, a.n_cmp[b], a.width, a.stride), a.n_max);
      for (int j = threadIdx.x; j < nv; j += 128)
        if (j < kAtRowCap) sm.rows[j] = j;
      base = nv;
    } else {
      __shared__ int scan_tmp[4];
      const int* sel = a.idx + (size_t)row_q * a.topk;
      constexpr int kMaxK = kAtRowCap / 128;
      int jv[kMaxK];
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {  // all loads in flight at once
        const int i = k * 128 + threadIdx.x;
        jv[k] = i < a.topk ? sel[i] : -1;
      }
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {
        if (k * 128 >= a.topk) break;
        int j = jv[k];
        if (j >= a.n_max) {
          report_error(CSA_ERR_DEVICE_BOUNDS);
          j = -1;
        }
        const int v = j >= 0 ? 1 : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += n;
        }
        if (lane == 31) scan_tmp[warp] = x;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        int off = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int c = scan_tmp[w];
          off += w < warp ? c : 0;
          tot += c;
        }
        if (v && base + off + x - 1 < kAtRowCap) sm.rows[base + off + x - 1] = j;
        base += tot;
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
    }
    {
      const int rp0 = a.raw_pos0[b];
      const int w_lo = max(max(0, t - a.window + 1), rp0);
      const int w_hi = min(t, rp0 + min(a.n_raw[b], a.raw_max) - 1);
      const int n_win = (a.window > 0 && w_hi >= w_lo) ? w_hi - w_lo + 1 : 0;
      for (int u = threadIdx.x; u < n_win; u += 128)
        if (base + u < kAtRowCap) sm.rows[base + u] = a.n_max + (w_lo - rp0) + u;
      if (threadIdx.x == 0) sm.n_rows = min(base + n_win, kAtRowCap);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // rope table + rows written
    mbar_arrive(&sm.rows_ready);
  }

  // this split's rows (rows_ready orders the reads after the writes)
  const bool rows_ok = mbar_wait(&sm.rows_ready, 0, abortp);
  const int R = rows_ok ? sm.n_rows : 0;
  const int r_lo = (int)((long long)R * split / a.splits);
  const int r_hi = (int)((long long)R * (split + 1) / a.splits);
  const int nrow = r_hi - r_lo;
  const int ntile = (nrow + kAtTile - 1) / kAtTile;

  if (warp < 4) {
    const int head = warp * 32 + lane;  // TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // ---- q: other half from staging to TMEM, RoPE on the rotated dims,
    //      rounded to bf16
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_tma, 0, abortp));
    if (ok) {
#pragma unroll 1
      for (int sbi = 0; sbi < 8; ++sbi) {
        const bool own = (sbi >> 2) == half;
        const int d0 = sbi * 64;
        const bool rot = d0 + 64 > rope0;
        if (own && !rot) continue;
        uint8_t* blk = own ? sm.q_own[sbi & 3] : q_stage + (sbi & 3) * (kAtHeads * 128);
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = *reinterpret_cast<const uint4*>(blk + swz(head, u));
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        if (rot) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int d = d0 + 2 * e;
            if (d >= rope0) {
              const int i = (d - rope0) >> 1;
              __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162*>(&w[e]);
              const float2 f = __bfloat1622float2(h2);
              w[e] = pack_bf16x2(f.x * sm.cs[i] - f.y * sm.sn[i], f.x * sm.sn[i] + f.y * sm.cs[i]);
            }
          }
        }
        if (own) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(blk + swz(head, u)) =
                make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        } else {
          const uint32_t col = (uint32_t)((sbi & 3) * 32);
          uint32_t r16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r16[e] = w[e];
          tmem_st16(t_q + lane_base + col, r16);
#pragma unroll
          for (int e = 0; e < 16; ++e) r16[e] = w[16 + e];
          tmem_st16(t_q + lane_base + col + 16, r16);
        }
      }
    }
    tmem_wait_st();
    fence_proxy_async();
    tc_fence_before();
    mbar_arrive(&sm.q_ready);

    // ---- online softmax over the tiles
    float m_run = -INFINITY, l_run = 0.f;
    for (int i = 0; i < ntile && ok; ++i) {
      const int sb = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], ph, abortp));
      if (!ok) break;
      tc_fence_after();
      const int valid = min(kAtTile, nrow - i * kAtTile);
      float z[64];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tmem_ld32(t_s + lane_base + (uint32_t)(sb * 64 + hh * 32), r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) z[hh * 32 + e] = __uint_as_float(r[e]) * a.scale_log2;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        if (e >= valid) z[e] = -INFINITY;
        mt = fmaxf(mt, z[e]);
      }
      if (mt > m_run + kAtRescaleLog2 || m_run == -INFINITY) {
        if (i > 0) {
          // O holds P V of earlier tiles: wait for the last PV, then rescale
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(i - 1) & 1],
                                                 (uint32_t)((i - 1) >> 1) & 1u, abortp));
          if (!ok) break;
          tc_fence_after();
          const float alpha = exp2f(m_run - mt);
#pragma unroll 1
          for (int cc = 0; cc < 256; cc += 32) {
            uint32_t r[32];
            tmem_ld32(t_o + lane_base + (uint32_t)cc, r);
            tmem_wait_ld();
            uint32_t w16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w16[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st16(t_o + lane_base + (uint32_t)cc, w16);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              w16[e] = __float_as_uint(__uint_as_float(r[16 + e]) * alpha);
            tmem_st16(t_o + lane_base + (uint32_t)cc + 16, w16);
          }
          l_run *= alpha;
        }
        m_run = mt;
      }
      uint32_t pk[32];
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = exp2f(z[2 * e] - m_run), p1 = exp2f(z[2 * e + 1] - m_run);
        __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
        const float2 back = __bfloat1622float2(pb);
        psum += back.x + back.y;
        pk[e] = *reinterpret_cast<uint32_t*>(&pb);
      }
      l_run += psum;
      uint32_t w16[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) w16[e] = pk[e];
      tmem_st16(t_s + lane_base + (uint32_t)(sb * 64), w16);
#pragma unroll
      for (int e = 0; e < 16; ++e) w16[e] = pk[16 + e];
      tmem_st16(t_s + lane_base + (uint32_t)(sb * 64 + 16), w16);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[sb]);
    }
    // ---- epilogue
    if (ok && ntile > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(ntile - 1) & 1],
                                             (uint32_t)((ntile - 1) >> 1) & 1u, abortp));
    if (ok) {
      tc_fence_after();
      const float sink_l2 = a.sink[head] * 1.4426950408889634f;
      if (a.splits == 1) {
        const float mm = fmaxf(m_run, sink_l2);
        const float den = (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - mm)) +
                          exp2f(sink_l2 - mm);
        const float scl = (m_run == -INFINITY || !(den > 0.f)) ? 0.f : exp2f(m_run - mm) / den;
        __nv_bfloat16* dst = a.out + ((size_t)row_q * kAtHeads + head) * kAtDim + half * 256;
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 32) {
          float o[32];
          if (ntile > 0) {
            uint32_t r[32];
            tmem_ld32(t_o + lane_base + (uint32_t)cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(r[e]) * scl;
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
          }
          const int d0 = half * 256 + cc;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int d = d0 + e;
            if (d >= rope0) {  // inverse rotation at -t
              const int ii = (d - rope0) >> 1;
              const float x0 = o[e], x1 = o[e + 1];
              o[e] = x0 * sm.cs[ii] + x1 * sm.sn[ii];
              o[e + 1] = -x0 * sm.sn[ii] + x1 * sm.cs[ii];
            }
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            d4[u] = make_uint4(pack_bf16x2(o[8 * u], o[8 * u + 1]),
                               pack_bf16x2(o[8 * u + 2], o[8 * u + 3]),
                               pack_bf16x2(o[8 * u + 4], o[8 * u + 5]),
                               pack_bf16x2(o[8 * u + 6], o[8 * u + 7]));
        }
      } else {
        const size_t unit = ((size_t)row_q * a.splits + split) * 2 + half;
        float* po = a.part_o + (unit * kAtHeads + head) * 256;
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 32) {
          float4* d4 = reinterpret_cast<float4*>(po + cc);
          if (ntile > 0) {
            uint32_t r[32];
            tmem_ld32(t_o + lane_base + (uint32_t)cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 8; ++u)
              d4[u] = make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                                  __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3]));
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) d4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float* pml = a.part_ml + unit * 2 * kAtHeads;
        pml[head] = m_run;
        pml[kAtHeads + head] = l_run;
      }
    }
  } else if (warp < 8) {
    // ======================= gather producers (128 threads)
    const int pt = threadIdx.x - 128;
    const __nv_bfloat16* cmp = a.kv_cmp + (size_t)b * a.n_max * kAtDim;
    const __nv_bfloat16* raw = a.kv_raw + (size_t)b * a.raw_max * kAtDim;
    int n1 = 0, n2 = 0;  // chunks issued into each ring
    bool okp = rows_ok;
    bool staged = false;  // q staging slots handed back
    for (int i = 0; i < ntile && okp; ++i) {
      const int tb = i & 1;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (pt < kAtTile) {
        const int r = r_lo + i * kAtTile + pt;
        const __nv_bfloat16* p = nullptr;
        if (r < r_hi) {
          const int id = sm.rows[r];
          p = id < a.n_max ? cmp + (size_t)id * kAtDim : raw + (size_t)(id - a.n_max) * kAtDim;
        }
        sm.row_ptr[tb][pt] = p;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      for (int ck = 0; ck < 4; ++ck) {
        const bool own = ck >= 2;
        const int chunk = own ? own0 + (ck - 2) : oth0 + ck;
        int slot;
        uint64_t* full;
        uint8_t* base;
        // one elected thread waits for the slot; the decision is shared so
        // that all 128 producers leave the loop together
        if (!own) {
          slot = n1 % kAtR1;
          if (pt == 0)
            sm.prod_ok = mbar_wait(&sm.r1_empty[slot], ((uint32_t)(n1 / kAtR1) & 1u) ^ 1u, abortp);
          full = &sm.r1_full[slot];
          base = sm.r1[slot];
          ++n1;
        } else {
          slot = n2 % kAtR2;
          if (pt == 0) {
            bool w = mbar_wait(&sm.r2_empty[slot], ((uint32_t)(n2 / kAtR2) & 1u) ^ 1u, abortp);
            if (w && !staged && slot >= kAtR2 - 4) {  // slot still holds q staging
              w = mbar_wait(&sm.q_ready, 0, abortp);
              staged = true;
            }
            sm.prod_ok = w;
          }
          full = &sm.r2_full[slot];
          base = sm.r2[slot];
          ++n2;
        }
        asm volatile("bar.sync 2, 128;" ::: "memory");
        okp = sm.prod_ok != 0;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (!okp) break;
        const uint32_t dst0 = smem_u32(base);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int piece = pt + 128 * k;  // 0..1023
          const int r = piece >> 4;        // row in tile
          const int q16 = piece & 15;      // 16 B unit within the 256 B chunk
          const __nv_bfloat16* rp = sm.row_ptr[tb][r];
          const void* src = rp ? (const void*)(rp + chunk * 128 + q16 * 8) : (const void*)a.q;
          const uint32_t dst = dst0 + (uint32_t)((q16 >> 3) * (kAtChunkBytes / 2)) +
                               swz(r, q16 & 7);
          cp_async16(dst, src, rp != nullptr);
        }
        cp_async_arrive(full);  // completes the chunk's phase when the copies land
      }
    }
    cp_async_wait_all();
  } else if (warp == 8 && lane == 0) {
    // ======================= MMA issuer
    constexpr uint32_t id_qk = idesc_bf16_f32(128, kAtTile);
    constexpr uint32_t id_pv = idesc_bf16_f32(128, 128, 0, 1);
    int c1 = 0, c2 = 0;  // chunks consumed per ring
    int own_slot[2][2];
    int last_pv = -1, last_s = -1;
    bool okm = rows_ok && mbar_wait(&sm.q_ready, 0, abortp);
    tc_fence_after();
    const uint32_t qs = smem_u32(sm.q_own[0]);
    auto issue_pv = [&](int j) -> bool {
      const int sb = j & 1;
      if (!mbar_wait(&sm.p_full[sb], (uint32_t)(j >> 1) & 1u, abortp)) return false;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kAtTile / 16; ++ks) {
#pragma unroll
        for (int oc = 0; oc < 2; ++oc) {
          const uint32_t vb = smem_u32(sm.r2[own_slot[sb][oc]]) + (uint32_t)(ks * 16 * 128);
          const uint64_t bd = sw128_desc(vb, kAtChunkBytes / 2, 1024);
          mma_ts(t_o + (uint32_t)(oc * 128), t_s + (uint32_t)(sb * 64 + ks * 8), bd, id_pv,
                 (j > 0 || ks > 0) ? 1u : 0u);
        }
      }
      tc_commit(&sm.r2_empty[own_slot[sb][0]]);
      tc_commit(&sm.r2_empty[own_slot[sb][1]]);
      tc_commit(&sm.pv_done[sb]);
      last_pv = j;
      return true;
    };
    for (int i = 0; i < ntile && okm; ++i) {
      const int sb = i & 1;
      if (i >= 2) {  // P(i-2) lives in S[sb]: its PV must have finished
        okm = mbar_wait(&sm.pv_done[sb], (uint32_t)((i - 2) >> 1) & 1u, abortp);
        if (!okm) break;
        tc_fence_after();
      }
      // S(i) = Q K_i^T over the four 128-dim chunks (other half first)
      for (int ck = 0; ck < 4 && okm; ++ck) {
        const bool own = ck >= 2;
        int slot;
        if (!own) {
          slot = c1 % kAtR1;
          okm = mbar_wait(&sm.r1_full[slot], (uint32_t)(c1 / kAtR1) & 1u, abortp);
          ++c1;
        } else {
          slot = c2 % kAtR2;
          okm = mbar_wait(&sm.r2_full[slot], (uint32_t)(c2 / kAtR2) & 1u, abortp);
          own_slot[sb][ck - 2] = slot;
          ++c2;
        }
        if (!okm) break;
        // the chunk was written by cp.async (generic proxy); the MMA reads it
        // through the async proxy
        fence_proxy_async();
        tc_fence_after();
        const uint32_t kb = smem_u32(own ? sm.r2[slot] : sm.r1[slot]);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bd = sw128_desc(kb + (uint32_t)((ks >> 2) * (kAtChunkBytes / 2) +
                                                         (ks & 3) * 32), 16, 1024);
          const uint32_t acc = (ck | ks) != 0 ? 1u : 0u;
          if (!own) {
            mma_ts(t_s + (uint32_t)(sb * 64), t_q + (uint32_t)(ck * 64 + ks * 8), bd, id_qk, acc);
          } else {
            const int sbq = (ck - 2) * 2 + (ks >> 2);
            const uint64_t ad = sw128_desc(qs + (uint32_t)(sbq * kAtHeads * 128 + (ks & 3) * 32),
                                           16, 1024);
            mma_ss(t_s + (uint32_t)(sb * 64), ad, bd, id_qk, acc);
          }
        }
        if (!own) tc_commit(&sm.r1_empty[slot]);
      }
      if (!okm) break;
      tc_commit(&sm.s_full[sb]);
      last_s = i;
      if (i >= 1) okm = issue_pv(i - 1);
    }
    if (okm && ntile > 0) okm = issue_pv(ntile - 1);
    // TMEM is freed only after the last MMAs have landed
    int never = 0;
    if (last_s >= 0)
      mbar_wait(&sm.s_full[last_s & 1], (uint32_t)(last_s >> 1) & 1u, &never, 100000000ull);
    if (last_pv >= 0)
      mbar_wait(&sm.pv_done[last_pv & 1], (uint32_t)(last_pv >> 1) & 1u, &never, 100000000ull);
  }
  // every copy issued into shared memory has landed before the CTA may exit
  if (warp == 4 && lane == 0) {
    int never = 0;
    mbar_wait(&sm.q_tma, 0, &never, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Split-KV merge: per (query token, head, dim) the partials (m_s, l_s, O_s)
// of every split, the sink and the inverse output rotation.  One block per
// (query token, output half, 8 heads); a thread owns 8 consecutive dims.
__global__ void __launch_bounds__(256) k_attn_combine(AttnTcArgs a) {
  __shared__ float cs[256], sn[256];
  const int row_q = blockIdx.x;
  const int half = blockIdx.y;
  const int head = blockIdx.z * 8 + (threadIdx.x >> 5);
  const int c0 = (threadIdx.x & 31) * 8;  // dims half*256 + c0 .. + 7
  const int t = a.q_pos[row_q];
  const int rope0 = kAtDim - a.rope_dim;
  const int S = a.splits;
  if (threadIdx.x < a.rope_dim / 2) {
    float c, s;
    rope_cos_sin(-(long long)t, threadIdx.x, a.rope_dim, a.theta, &c, &s);
    cs[threadIdx.x] = c;
    sn[threadIdx.x] = s;
  }
  __syncthreads();
  const float sink_l2 = a.sink[head] * 1.4426950408889634f;
  float M = sink_l2;
  for (int s = 0; s < S; ++s) {
    const size_t unit = ((size_t)row_q * S + s) * 2 + half;
    M = fmaxf(M, a.part_ml[unit * 2 * kAtHeads + head]);
  }
  float L = exp2f(sink_l2 - M);
  float o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) o[e] = 0.f;
  for (int s = 0; s < S; ++s) {
    const size_t unit = ((size_t)row_q * S + s) * 2 + half;
    const float m = a.part_ml[unit * 2 * kAtHeads + head];
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    L += a.part_ml[unit * 2 * kAtHeads + kAtHeads + head] * w;
    const float4* src = reinterpret_cast<const float4*>(a.part_o + (unit * kAtHeads + head) * 256 + c0);
    const float4 v0 = src[0], v1 = src[1];
    o[0] += v0.x * w; o[1] += v0.y * w; o[2] += v0.z * w; o[3] += v0.w * w;
    o[4] += v1.x * w; o[5] += v1.y * w; o[6] += v1.z * w; o[7] += v1.w * w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float x0 = o[e] * inv, x1 = o[e + 1] * inv;
    const int d = half * 256 + c0 + e;
    if (d >= rope0) {
      const float c = cs[(d - rope0) >> 1], s = sn[(d - rope0) >> 1];
      const float y0 = x0 * c - x1 * s, y1 = x0 * s + x1 * c;
      x0 = y0;
      x1 = y1;
    }
    o[e] = x0;
    o[e + 1] = x1;
  }
  *reinterpret_cast<uint4*>(a.out + ((size_t)row_q * kAtHeads + head) * kAtDim + half * 256 + c0) =
      make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                 pack_bf16x2(o[6], o[7]));
}

}  // namespace csa
