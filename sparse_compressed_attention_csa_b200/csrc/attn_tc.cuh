// Steps 3 and 4 on tensor cores, for the measured shape (128 query heads x
// 512 dims, bf16): shared-KV MQA over the selected compressed entries (CSA)
// or every visible entry (HCA), plus the raw window, with the per-head sink
// and partial RoPE ("Compressed Sparse Attention", "Heavily Compressed
// Attention", "Partial RoPE" and "Output gate + sink" rows).
//
// One query token = one MMA M of 128 heads.  Its output O (128 x 512 fp32)
// alone would fill all of TMEM (128 lanes x 512 columns), so each query is
// split over NQ CTAs by output dims: CTA `part` owns d_v columns
// [part * 512/NQ, (part + 1) * 512/NQ) and computes S = Q K^T itself.
//
//   NQ = 2 (many queries: prefill; S recomputed twice)
//     TMEM  O [0,256) | S0 [256,320) | S1 [320,384) | Q other half [384,512)
//     SMEM  Q own half (64 KB) | ring of 9 chunks | row list
//   NQ = 4 (few queries: decode; S recomputed four times, but the whole of Q
//           sits in TMEM, which frees shared memory for a deeper gather ring)
//     TMEM  O [0,128) | S0 [128,192) | S1 [192,256) | Q [256,512)
//     SMEM  ring of 13 chunks | row list
//
// Q is rotated at the query position and rounded to bf16 once, after one TMA
// load of [128 heads][64 dims] boxes.  KV rows are gathered 64 at a time by
// 128 threads with 16-byte cp.async into 128B-swizzled shared memory (the
// gather reaches full bandwidth only with many requests in flight, which
// many issuing threads sustain and one-warp TMA gathers do not).  A row
// streams as four 128-dim chunks through a FIFO ring; chunks outside the
// CTA's output dims feed only S and are released right after it, the CTA's
// own chunks then serve as V for the PV product and are held until it
// completes.  The row list holds selected entries, then window rows, each
// padded to a multiple of 4 with masked rows.
//
//   warp 8 (one thread): MMAs   S(i) = Q K_i^T  (N = 64, K = 512)
//                               O   += P(i-1) V(i-1)  (A = P from TMEM, N = 128 per chunk)
//   warps 4-7: gather producers (q by TMA, rows by cp.async, no barriers)
//   warps 0-3: one head per thread (= TMEM lane): online softmax in the
//              log2 domain with a lazy rescale (only when the running max
//              grows by more than 2^8), P written back over S as bf16,
//              epilogue with the sink, the inverse output rotation and the
//              store (or split-KV partials for k_attn_combine).
// Every mbarrier wait is bounded; a timeout records CSA_ERR_DEVICE_TIMEOUT
// and the CTA winds down, frees TMEM and exits.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kAtHeads = 128;
constexpr int kAtDim = 512;
constexpr int kAtTile = 64;                       // KV rows per S tile (MMA N)
constexpr int kAtChunkBytes = kAtTile * 128 * 2;  // 64 rows x 128 dims bf16
constexpr int kAtSubBytes = kAtHeads * 128;       // q box: [128 heads][64 dims]
constexpr int kAtRowCap = 2048;                   // rows per query token
constexpr int kAtMaxRope = 128;                   // rotated dims supported
constexpr int kAtMaxSlots = 13;
constexpr int kAtMaxSplits = 16;                  // split-KV parts per query token
constexpr int kAtThreads = 288;
constexpr float kAtRescaleLog2 = 8.0f;

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
  int splits;
  __nv_bfloat16* out;  // splits == 1
  float* part_o;       // splits > 1: [B*Tq][splits][NQ][512/NQ/32][8][128][4]
  float* part_ml;      // [B*Tq][splits][NQ][2][128]  (m, l)
  int* arrive;         // [B*Tq][NQ] split arrivals, zero before the launch
  double freq[kAtMaxRope / 2];  // RoPE frequencies theta^(-2i/rope_dim)
};

struct AtMisc {
  int rows[kAtRowCap];  // gather row coordinates
  float cs[kAtMaxRope / 2], sn[kAtMaxRope / 2];
  uint64_t full[kAtMaxSlots], empty[kAtMaxSlots];
  uint64_t s_full[2], p_full[2], pv_done[2], q_tma, q_ready, rows_ready, rope_ready, merge_bar;
  uint32_t tmem_base;
  int n_rows;  // padded rows (multiple of 4)
  int n_sel;   // selected rows (valid rows [0, n_sel))
  int n_win;   // window rows (valid rows [pad4(n_sel), pad4(n_sel) + n_win))
  int abort_flag;
  int scan_tmp[4];
};

template <int NQ>
struct AtLayout {
  static constexpr int kSlots = NQ == 2 ? 9 : 13;
  static constexpr int kOwnChunks = 4 / NQ;         // 128-dim chunks of output dims
  static constexpr int kOCols = kAtDim / NQ;        // output dims (and O columns)
  static constexpr int kQOwnSub = NQ == 2 ? 4 : 0;  // q sub-blocks kept in shared memory
  static constexpr int kQStage = 8 - kQOwnSub;      // q sub-blocks staged for TMEM
  static constexpr int kRingOff = kQOwnSub * kAtSubBytes;
  static constexpr int kMiscOff = kRingOff + kSlots * kAtChunkBytes;
  static constexpr size_t kBytes = (size_t)kMiscOff + sizeof(AtMisc);
  static constexpr uint32_t kTmemS = kOCols;         // S0, S1: 2 x 64 columns
  static constexpr uint32_t kTmemQ = kOCols + 128;   // Q chunks held in TMEM
};
static_assert(AtLayout<2>::kBytes + 1024 <= 232448, "shared memory budget (NQ = 2)");
static_assert(AtLayout<4>::kBytes + 1024 <= 232448, "shared memory budget (NQ = 4)");

// 2^x by the hardware approximation (relative error ~2^-22; the softmax
// weights are rounded to bf16 right after).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
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

// cos / sin of pos * freq: the angle is reduced modulo 2 pi in double
// precision (2 pi split in two parts), then taken in fp32.
__device__ __forceinline__ void rope_cs_reduced(long long pos, double freq, float* c, float* s) {
  const double x = (double)pos * freq;
  const double k = rint(x * 0.15915494309189535);
  double r = fma(-k, 6.283185307179586, x);
  r = fma(-k, 2.4492935982947064e-16, r);
  sincosf((float)r, s, c);
}

template <bool kHca, int NQ>
__global__ void __launch_bounds__(kAtThreads, 1)
    k_attn_tc(AttnTcArgs a, const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_out) {
  using namespace sm100;
  using Lay = AtLayout<NQ>;
  constexpr int kSlots = Lay::kSlots;
  constexpr int kOwn = Lay::kOwnChunks;
  constexpr int kOCols = Lay::kOCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base_ptr = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
  uint8_t* q_own = base_ptr;                 // kQOwnSub x [128][128 B]
  uint8_t* ring = base_ptr + Lay::kRingOff;  // kSlots x 16 KB
  AtMisc& sm = *reinterpret_cast<AtMisc*>(base_ptr + Lay::kMiscOff);

  const int part = blockIdx.x % NQ;
  const int split = blockIdx.x / NQ;
  const int row_q = blockIdx.y;  // b * Tq + tq
  const int b = row_q / a.Tq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = a.q_pos[row_q];
  const int rope0 = kAtDim - a.rope_dim;
  // 128-dim chunks in streaming order: the others first, then the own ones
  // (own chunks: dims part * kOCols ..)
  const int own0 = part * kOwn;
  int chunk_of[4];
  {
    int w = 0;
    for (int c = 0; c < 4; ++c)
      if (c < own0 || c >= own0 + kOwn) chunk_of[w++] = c;
    for (int c = 0; c < kOwn; ++c) chunk_of[w++] = own0 + c;
  }
  // q sub-block sb (64 dims) lives in shared memory (own half, NQ = 2) or in
  // TMEM at column 32 * q_tidx(sb); TMEM-bound sub-blocks are staged in the
  // last ring slots
  auto q_in_smem = [&](int sb) { return NQ == 2 && (sb >> 2) == part; };
  auto q_tidx = [&](int sb) { return NQ == 2 ? (sb & 3) : sb; };
  uint8_t* q_stage = ring + (kSlots - Lay::kQStage) * kAtChunkBytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 128);
      mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.pv_done[i], 1);
    }
    mbar_init(&sm.q_tma, 1);
    mbar_init(&sm.q_ready, 128);
    mbar_init(&sm.rows_ready, 128);
    mbar_init(&sm.rope_ready, 32);
    mbar_init(&sm.merge_bar, 1);
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
  const uint32_t t_o = tmem, t_s = tmem + Lay::kTmemS, t_q = tmem + Lay::kTmemQ;
  volatile int* abortp = &sm.abort_flag;

  if (warp == 4 && lane == 0) {
    // q of this token: 8 boxes of [128 heads][64 dims], 128B swizzle
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_out);
    mbar_arrive_expect_tx(&sm.q_tma, kAtHeads * kAtDim * 2);
    for (int sb = 0; sb < 8; ++sb) {
      uint8_t* dst = q_in_smem(sb) ? q_own + (sb & 3) * kAtSubBytes
                                   : q_stage + q_tidx(sb) * kAtSubBytes;
      tma_load_2d(dst, &tm_q, &sm.q_tma, sb * 64, row_q * kAtHeads);
    }
  }
  if (warp == 8) {
    // RoPE table at the query position (this warp only issues MMAs once q is
    // in place)
    for (int i = lane; i < a.rope_dim / 2; i += 32) {
      float c, s;
      rope_cs_reduced(t, a.freq[i], &c, &s);
      sm.cs[i] = c;
      sm.sn[i] = s;
    }
    mbar_arrive(&sm.rope_ready);
  }

  if (warp >= 4 && warp < 8) {
    // ======================= row list (warps 4-7, while warps 0-3 stage q):
    // gather coordinates of the selected (or visible) entries, then the
    // window's raw rows, each part padded to a multiple of 4 rows
    const int tid = threadIdx.x - 128;
    const int cmp_y0 = b * a.n_max;    // row 0 of this sequence in kv_cmp
    const int raw_y0 = b * a.raw_max;  // row 0 of this sequence in kv_raw
    int base = 0;
    if (kHca) {
      const int nv = min(min(n_visible(t, a.n_cmp[b], a.width, a.stride), a.n_max), kAtRowCap);
      for (int j = tid; j < nv; j += 128) sm.rows[j] = cmp_y0 + j;
      base = nv;
    } else {
      const int* sel = a.idx + (size_t)row_q * a.topk;
      constexpr int kMaxK = kAtRowCap / 128;
      int jv[kMaxK];
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {  // every load in flight at once
        const int i = k * 128 + tid;
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
        if (lane == 31) sm.scan_tmp[warp - 4] = x;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        int off = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int c = sm.scan_tmp[w];
          off += w < warp - 4 ? c : 0;
          tot += c;
        }
        if (v && base + off + x - 1 < kAtRowCap) sm.rows[base + off + x - 1] = cmp_y0 + j;
        base += tot;
        asm volatile("bar.sync 2, 128;" ::: "memory");
      }
      base = min(base, kAtRowCap);
    }
    const int n_sel = base;
    const int ps = (n_sel + 3) & ~3;
    for (int k = n_sel + tid; k < ps; k += 128) sm.rows[k] = cmp_y0;  // masked padding
    {
      const int rp0 = a.raw_pos0[b];
      const int w_lo = max(max(0, t - a.window + 1), rp0);
      const int w_hi = min(t, rp0 + min(a.n_raw[b], a.raw_max) - 1);
      int n_win = (a.window > 0 && w_hi >= w_lo) ? w_hi - w_lo + 1 : 0;
      n_win = max(0, min(n_win, kAtRowCap - ps));
      const int pw = (n_win + 3) & ~3;
      for (int u = tid; u < pw; u += 128)
        sm.rows[ps + u] = raw_y0 + (w_lo - rp0) + (u < n_win ? u : 0);
      if (tid == 0) {
        sm.n_sel = n_sel;
        sm.n_win = n_win;
        sm.n_rows = ps + pw;
      }
    }
    asm volatile("bar.sync 2, 128;" ::: "memory");  // rows written
    mbar_arrive(&sm.rows_ready);
  }

  // this split's rows, in groups of 4 (each role waits for rows_ready
  // before reading the list)
  bool rows_ok = false;
  int r_lo = 0, r_hi = 0, nrow = 0, ntile = 0;
  auto load_split = [&]() {
    rows_ok = mbar_wait(&sm.rows_ready, 0, abortp);
    const int G = rows_ok ? sm.n_rows / 4 : 0;
    r_lo = 4 * (int)((long long)G * split / a.splits);
    r_hi = 4 * (int)((long long)G * (split + 1) / a.splits);
    nrow = r_hi - r_lo;
    ntile = (nrow + kAtTile - 1) / kAtTile;
  };

  if (warp < 4) {
    // ======================= softmax / epilogue warps
    const int head = warp * 32 + lane;  // TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // ---- q: staged sub-blocks to TMEM, RoPE on the rotated dims, bf16
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_tma, 0, abortp) &&
                                              mbar_wait(&sm.rope_ready, 0, abortp));
    if (ok) {
#pragma unroll 1
      for (int sb = 0; sb < 8; ++sb) {
        const bool in_smem = q_in_smem(sb);
        const int d0 = sb * 64;
        const bool rot = d0 + 64 > rope0;
        if (in_smem && !rot) continue;
        uint8_t* blk = in_smem ? q_own + (sb & 3) * kAtSubBytes
                               : q_stage + q_tidx(sb) * kAtSubBytes;
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
        if (in_smem) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(blk + swz(head, u)) =
                make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        } else {
          const uint32_t col = (uint32_t)(q_tidx(sb) * 32);
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
    load_split();
    ok = ok && __all_sync(0xffffffffu, rows_ok);

    // ---- online softmax over the tiles
    const int n_sel = sm.n_sel, ps = (n_sel + 3) & ~3, pe = ps + sm.n_win;
    float m_run = -INFINITY, l_run = 0.f;
    for (int i = 0; i < ntile && ok; ++i) {
      const int sb = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], ph, abortp));
      if (!ok) break;
      tc_fence_after();
      const int g0 = r_lo + i * kAtTile;  // list index of row 0 of the tile
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
        const int g = g0 + e;
        const bool valid = g < r_hi && (g < n_sel || (g >= ps && g < pe));
        if (!valid) z[e] = -INFINITY;
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
          for (int cc = 0; cc < kOCols; cc += 32) {
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
        const float p0 = ex2_approx(z[2 * e] - m_run), p1 = ex2_approx(z[2 * e + 1] - m_run);
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
    {  // all four softmax warps agree before the named barriers below
      uint32_t all;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
          "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(all)
          : "r"(ok ? 1u : 0u)
          : "memory");
      ok = all != 0;
    }
    if (ok) {
      tc_fence_after();
      // Shared memory is idle once the last PV has landed (q's own half and
      // the ring are one contiguous block).  It holds, for a split-KV merge,
      // one other split's partial O (pbuf, in its global layout) and, for
      // the output, the bf16 tile of this CTA's dims as kOCols / 64 TMA boxes
      // of [128 heads][128 B], 128B-swizzled.
      constexpr int kPartBytes = kAtHeads * kOCols * 4;
      constexpr int kOutBoxes = kOCols / 64;
      static_assert(kPartBytes + kOutBoxes * kAtSubBytes + 2 * kAtMaxSplits * kAtHeads * 4 <=
                        Lay::kMiscOff,
                    "epilogue buffers exceed the idle shared memory");
      uint8_t* pbuf = base_ptr;
      uint8_t* obuf = base_ptr + kPartBytes;
      const float sink_l2 = a.sink[head] * 1.4426950408889634f;
      const int S = a.splits;
      const size_t unit0 = (size_t)row_q * S * NQ + part;  // unit of split s: unit0 + s * NQ
      // Partial O layout per unit: [slab of 32 dims][16-byte unit u][head][4
      // floats], so that a warp's 16-byte accesses at one (slab, u) are
      // contiguous.
      auto part_off = [&](int cc, int u) { return ((size_t)((cc / 32) * 8 + u) * kAtHeads + head) * 4; };
      // One pass over the 32-column slabs.  Terms src * w, in split order:
      // this CTA's O (TMEM; zero without tiles) and/or the partial in pbuf
      // (`buf_first`: the pbuf term comes first).  acc = terms (`first`) or
      // acc + terms, the running sum kept in TMEM columns [t_s, t_s +
      // kOCols) (S and q are dead by now).  mode 0: acc back to TMEM; 1: out
      // as this split's fp32 partial; 2: rotated back at -t, rounded to bf16
      // and stored through TMA.  Every product and sum is rounded on its own,
      // in split order, so a merge does not depend on which split performs
      // it.
      const uint32_t t_acc = t_s;
      auto slab_pass = [&](bool use_own, float w_own, bool use_buf, float w_buf, bool buf_first,
                           bool first, int mode) {
#pragma unroll 1
        for (int cc = 0; cc < kOCols; cc += 32) {
          float o[32];
          bool have = !first;
          if (have) {
            uint32_t r[32];
            tmem_ld32(t_acc + lane_base + (uint32_t)cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(r[e]);
          }
          auto add_own = [&]() {
            uint32_t r[32];
            if (ntile > 0) {
              tmem_ld32(t_o + lane_base + (uint32_t)cc, r);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = 0u;
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float tm = __fmul_rn(__uint_as_float(r[e]), w_own);
              o[e] = have ? __fadd_rn(o[e], tm) : tm;
            }
            have = true;
          };
          auto add_buf = [&]() {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float4 x =
                  *reinterpret_cast<const float4*>(pbuf + part_off(cc, u) * sizeof(float));
              const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const float tm = __fmul_rn(xs[v], w_buf);
                o[4 * u + v] = have ? __fadd_rn(o[4 * u + v], tm) : tm;
              }
            }
            have = true;
          };
          if (use_buf && buf_first) add_buf();
          if (use_own) add_own();
          if (use_buf && !buf_first) add_buf();
          if (mode == 0) {
            uint32_t w16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w16[e] = __float_as_uint(o[e]);
            tmem_st16(t_acc + lane_base + (uint32_t)cc, w16);
#pragma unroll
            for (int e = 0; e < 16; ++e) w16[e] = __float_as_uint(o[16 + e]);
            tmem_st16(t_acc + lane_base + (uint32_t)cc + 16, w16);
          } else if (mode == 1) {
            float* dst = a.part_o + (unit0 + (size_t)split * NQ) * kAtHeads * kOCols;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<float4*>(dst + part_off(cc, u)) =
                  make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
          } else {
            const int d0 = part * kOCols + cc;
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
            uint8_t* box = obuf + (cc / 64) * kAtSubBytes;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int u = ((cc & 63) >> 3) + j;
              *reinterpret_cast<uint4*>(box + swz(head, u)) =
                  make_uint4(pack_bf16x2(o[8 * j], o[8 * j + 1]), pack_bf16x2(o[8 * j + 2], o[8 * j + 3]),
                             pack_bf16x2(o[8 * j + 4], o[8 * j + 5]), pack_bf16x2(o[8 * j + 6], o[8 * j + 7]));
            }
          }
        }
        if (mode == 0) {
          tmem_wait_st();
          tc_fence_before();
        } else if (mode == 2) {
          fence_proxy_async_shared();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (threadIdx.x == 0) {
            for (int bx = 0; bx < kOutBoxes; ++bx)
              tma_store_2d(&tm_out, obuf + bx * kAtSubBytes, part * kOCols + bx * 64,
                           row_q * kAtHeads);
            bulk_commit();
            bulk_wait_read_all();
          }
        }
      };
      if (S == 1) {
        const float mm = fmaxf(m_run, sink_l2);
        const float den = (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - mm)) +
                          exp2f(sink_l2 - mm);
        const float scl =
            (m_run == -INFINITY || !(den > 0.f)) ? 0.f : exp2f(m_run - mm) / den;
        slab_pass(true, scl, false, 0.f, false, true, 2);
      } else {
        // split-KV: publish (m, l, O) of this split; the last split of the
        // (token, part) to finish merges all of them in split order (its
        // own O straight from TMEM) and resets the arrival counter
        float* pml = a.part_ml + (unit0 + (size_t)split * NQ) * 2 * kAtHeads;
        pml[head] = m_run;
        pml[kAtHeads + head] = l_run;
        slab_pass(true, 1.f, false, 0.f, false, true, 1);
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 0) {
          const int old = atomicAdd(a.arrive + (size_t)row_q * NQ + part, 1);
          sm.scan_tmp[0] = old == S - 1 ? 1 : 0;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (sm.scan_tmp[0]) {
          __threadfence();
          fence_proxy_async_global();  // the partials are read by bulk copies
          // (m, l) of every split for this thread's head, in one batch of loads
          float* mls = reinterpret_cast<float*>(obuf + kOutBoxes * kAtSubBytes);
#pragma unroll 4
          for (int sp = 0; sp < S; ++sp) {
            const float* ml = a.part_ml + (unit0 + (size_t)sp * NQ) * 2 * kAtHeads;
            mls[(2 * sp) * kAtHeads + head] = sp == split ? m_run : __ldcg(ml + head);
            mls[(2 * sp + 1) * kAtHeads + head] = sp == split ? l_run : __ldcg(ml + kAtHeads + head);
          }
          float M = sink_l2;
          for (int sp = 0; sp < S; ++sp) M = fmaxf(M, mls[(2 * sp) * kAtHeads + head]);
          float L = exp2f(sink_l2 - M);
          for (int sp = 0; sp < S; ++sp) {
            const float m = mls[(2 * sp) * kAtHeads + head];
            if (m != -INFINITY) L += mls[(2 * sp + 1) * kAtHeads + head] * exp2f(m - M);
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          auto weight = [&](int sp) {
            const float m = mls[(2 * sp) * kAtHeads + head];
            return m == -INFINITY ? 0.f : exp2f(m - M) * inv;
          };
          int loads = 0;
          bool okm = true;
          auto fetch = [&](int sp) -> bool {  // partial O of split sp into pbuf
            if (threadIdx.x == 0) {
              mbar_arrive_expect_tx(&sm.merge_bar, kPartBytes);
              bulk_load(pbuf, a.part_o + (unit0 + (size_t)sp * NQ) * kAtHeads * kOCols,
                        kPartBytes, &sm.merge_bar);
            }
            bool got = __all_sync(0xffffffffu,
                                  mbar_wait(&sm.merge_bar, (uint32_t)(loads & 1), abortp));
            ++loads;
            uint32_t all;  // the four warps agree before going on
            asm volatile(
                "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(all)
                : "r"(got ? 1u : 0u)
                : "memory");
            return all != 0;
          };
          // passes over the splits in order; this CTA's own O joins the pass
          // of its neighbour, so two splits take one pass and one copy
          bool first = true;
          for (int sp = 0; sp < S && okm;) {
            if (sp == split) {
              if (sp + 1 < S) {
                okm = fetch(sp + 1);
                if (!okm) break;
                slab_pass(true, weight(sp), true, weight(sp + 1), false, first,
                          sp + 2 == S ? 2 : 0);
                sp += 2;
              } else {
                slab_pass(true, weight(sp), false, 0.f, false, first, 2);
                sp += 1;
              }
            } else {
              okm = fetch(sp);
              if (!okm) break;
              const bool with_own = sp + 1 == split;
              const int next = sp + (with_own ? 2 : 1);
              slab_pass(with_own, with_own ? weight(sp + 1) : 0.f, true, weight(sp), true, first,
                        next == S ? 2 : 0);
              sp = next;
            }
            first = false;
            asm volatile("bar.sync 1, 128;" ::: "memory");  // pbuf free again
          }
          if (threadIdx.x == 0) a.arrive[(size_t)row_q * NQ + part] = 0;
        }
      }
    }
  } else if (warp < 8) {
    // ======================= gather producers (128 threads)
    // Chunk n (tile n / 4, part n % 4 in streaming order) goes to ring slot
    // n % kSlots.  Every thread waits for the slot itself and issues its own
    // 8 copies of each chunk (rows (pt >> 4) + 8 m, 16-byte unit pt & 15): no
    // barrier among the producers, so the copy issue never waits on the
    // slowest thread.  Rows past the split end are zero-filled (masked).
    load_split();
    const int pt = threadIdx.x - 128;
    const int q16 = pt & 15;
    const int r0 = pt >> 4;
    const int n_sel = sm.n_sel, ps = (n_sel + 3) & ~3;
    bool okp = rows_ok;
    bool staged = false;  // q staging slots handed back
    int n = 0;
    for (int i = 0; i < ntile && okp; ++i) {
      const __nv_bfloat16* rp[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int g = r_lo + i * kAtTile + r0 + 8 * m;
        rp[m] = nullptr;
        if (g < r_hi) {
          const int y = sm.rows[g];
          rp[m] = (g < ps ? a.kv_cmp : a.kv_raw) + (size_t)y * kAtDim;
        }
      }
      for (int ck = 0; ck < 4; ++ck, ++n) {
        const int chunk = chunk_of[ck];
        const int slot = n % kSlots;
        okp = mbar_wait_backoff(&sm.empty[slot], ((uint32_t)(n / kSlots) & 1u) ^ 1u, abortp);
        if (okp && !staged && slot >= kSlots - Lay::kQStage) {  // slot still holds q staging
          okp = mbar_wait_backoff(&sm.q_ready, 0, abortp);
          staged = true;
        }
        if (!okp) break;
        const uint32_t dst0 = smem_u32(ring + slot * kAtChunkBytes) +
                              (uint32_t)((q16 >> 3) * (kAtChunkBytes / 2));
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int r = r0 + 8 * m;
          const void* src = rp[m] ? (const void*)(rp[m] + chunk * 128 + q16 * 8) : (const void*)a.q;
          cp_async16(dst0 + swz(r, q16 & 7), src, rp[m] != nullptr);
        }
        cp_async_arrive(&sm.full[slot]);  // completes when the copies land
      }
    }
    cp_async_wait_all();
  } else if (warp == 8 && lane == 0) {
    // ======================= MMA issuer
    constexpr uint32_t id_qk = idesc_bf16_f32(128, kAtTile);
    constexpr uint32_t id_pv = idesc_bf16_f32(128, 128, 0, 1);
    int n = 0;  // chunks consumed
    int own_slot[2][kOwn];
    int last_pv = -1, last_s = -1;
    load_split();
    bool okm = rows_ok && mbar_wait(&sm.q_ready, 0, abortp);
    tc_fence_after();
    const uint32_t qs = smem_u32(q_own);
    auto issue_pv = [&](int j) -> bool {
      const int sb = j & 1;
      if (!mbar_wait(&sm.p_full[sb], (uint32_t)(j >> 1) & 1u, abortp)) return false;
      tc_fence_after();
#pragma unroll
      for (int oc = 0; oc < kOwn; ++oc) {
        const uint64_t vd0 =
            sw128_desc(smem_u32(ring + own_slot[sb][oc] * kAtChunkBytes), kAtChunkBytes / 2, 1024);
#pragma unroll
        for (int ks = 0; ks < kAtTile / 16; ++ks)
          mma_ts(t_o + (uint32_t)(oc * 128), t_s + (uint32_t)(sb * 64 + ks * 8),
                 vd0 + (uint64_t)((ks * 16 * 128) >> 4), id_pv, (j > 0 || ks > 0) ? 1u : 0u);
      }
#pragma unroll
      for (int oc = 0; oc < kOwn; ++oc) tc_commit(&sm.empty[own_slot[sb][oc]]);
      tc_commit(&sm.pv_done[sb]);
      last_pv = j;
      return true;
    };
    int pv_next = 0;  // next tile whose PV is still to be issued
    for (int i = 0; i < ntile && okm; ++i) {
      const int sb = i & 1;
      if (i >= 2) {  // P(i-2) lives in S[sb]: its PV must have finished
        if (pv_next <= i - 2) okm = issue_pv(pv_next++);
        if (!okm) break;
        okm = mbar_wait(&sm.pv_done[sb], (uint32_t)((i - 2) >> 1) & 1u, abortp);
        if (!okm) break;
        tc_fence_after();
      }
      // S(i) = Q K_i^T over the four 128-dim chunks (others first)
      for (int ck = 0; ck < 4 && okm; ++ck, ++n) {
        const int chunk = chunk_of[ck];
        const bool own = ck >= 4 - kOwn;
        const int slot = n % kSlots;
        okm = mbar_wait(&sm.full[slot], (uint32_t)(n / kSlots) & 1u, abortp);
        if (own) own_slot[sb][ck - (4 - kOwn)] = slot;
        if (!okm) break;
        // written by cp.async (generic proxy), read by the MMA (async proxy)
        fence_proxy_async();
        tc_fence_after();
        // descriptors: one per chunk, k steps by adding (offset >> 4) to the
        // start-address field
        const uint64_t bd0 = sw128_desc(smem_u32(ring + slot * kAtChunkBytes), 16, 1024);
        const int sbq0 = chunk * 2;
        if (!q_in_smem(sbq0)) {
          const uint32_t a0 = t_q + (uint32_t)(q_tidx(sbq0) * 32);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts(t_s + (uint32_t)(sb * 64), a0 + (uint32_t)((ks >> 2) * 32 + (ks & 3) * 8),
                   bd0 + (uint64_t)(((ks >> 2) * (kAtChunkBytes / 2) + (ks & 3) * 32) >> 4),
                   id_qk, (ck | ks) != 0 ? 1u : 0u);
        } else {
          const uint64_t ad0 = sw128_desc(qs + (uint32_t)((sbq0 & 3) * kAtSubBytes), 16, 1024);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(t_s + (uint32_t)(sb * 64),
                   ad0 + (uint64_t)(((ks >> 2) * kAtSubBytes + (ks & 3) * 32) >> 4),
                   bd0 + (uint64_t)(((ks >> 2) * (kAtChunkBytes / 2) + (ks & 3) * 32) >> 4),
                   id_qk, (ck | ks) != 0 ? 1u : 0u);
        }
        if (!own) tc_commit(&sm.empty[slot]);
        // the previous tile's PV goes in as soon as its P is ready
        if (pv_next == i - 1 && mbar_try_wait(&sm.p_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u))
          okm = issue_pv(pv_next++);
      }
      if (!okm) break;
      tc_commit(&sm.s_full[sb]);
      last_s = i;
    }
    while (okm && pv_next < ntile) okm = issue_pv(pv_next++);
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

}  // namespace csa
