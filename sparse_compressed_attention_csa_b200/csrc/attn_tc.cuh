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
//   NQ = 2 (the one the library launches; S recomputed twice)
//     TMEM  O [0,256) | S0 [256,320) | S1 [320,384) | Q other half [384,512)
//     SMEM  Q own half (64 KB) | ring of 9 chunks | row list
//   NQ = 4 (the template supports it; measured slower on every workload:
//           S recomputed four times, the whole of Q in TMEM, 13-chunk ring)
//     TMEM  O [0,128) | S0 [128,192) | S1 [192,256) | Q [256,512)
//     SMEM  ring of 13 chunks | row list
//
// Q is rotated at the query position and rounded to bf16 once, after one TMA
// load of [128 heads][64 dims] boxes.  KV rows are gathered 64 at a time by
// 128 threads with 16-byte cp.async into 128B-swizzled shared memory: in a
// random-row gather microbenchmark over all SMs (1 KB rows from a 1 GiB
// buffer) this reached 43 GB/s per SM, TMA tile::gather4 issued by one warp
// 15.5 and by four warps 38.7.  A row streams as four 128-dim chunks
// through a FIFO ring; chunks outside the CTA's output dims feed only S and
// are released right after it, the CTA's own chunks then serve as V for the
// PV product and are held until it completes.  The row list holds selected entries, then window rows, each
// padded to a multiple of 4 with masked rows.
//
//   warp 8 (one thread): MMAs   S(i) = Q K_i^T  (N = 64, K = 512)
//                               O   += P(i-1) V(i-1)  (A = P from TMEM, N = 128 per chunk)
//   warps 4-7: gather producers (q by TMA, rows by cp.async, no barriers)
//   warps 0-3: one head per thread (= TMEM lane): online softmax in the
//              log2 domain with a lazy rescale (only when the running max
//              grows by more than 2^8), P written back over S as bf16,
//              epilogue with the sink, the inverse output rotation and a
//              TMA store of the bf16 output.
//
// Split-KV (few query tokens): the S splits of one (token, part) form a
// thread-block cluster.  Each writes its (m, l) and partial O to the
// workspace; after a cluster barrier each CTA merges 1/S of the output dims
// over all splits.
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
constexpr int kAtMaxSplits = 8;                   // split-KV parts per query token (one cluster)
constexpr int kAtSlabBytes = kAtHeads * 32 * 4;    // 32 dims of fp32 O for 128 heads
constexpr int kAtOutBoxBytes = kAtHeads * 64;      // 32 dims of bf16 output for 128 heads
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
  float* part_o;       // splits > 1: [B*Tq][NQ][splits][512/NQ/32 slabs][8][128][4]
  float* part_ml;      // [B*Tq][NQ][splits][2][128]  (m, l)
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
// Idle shared memory the epilogue needs with S splits: (S - 1) partial slabs
// of the merged range per other split, plus the output boxes.
template <int NQ>
constexpr int at_epilogue_bytes() {
  int worst = (kAtDim / NQ / 32) * kAtOutBoxBytes;  // S = 1: every slab
  for (int S = 2; S <= kAtMaxSplits; ++S) {
    const int ns = (kAtDim / NQ / 32 + S - 1) / S;
    const int need = (S - 1) * ns * kAtSlabBytes + ns * kAtOutBoxBytes;
    worst = need > worst ? need : worst;
  }
  return worst;
}
static_assert(at_epilogue_bytes<2>() <= AtLayout<2>::kMiscOff, "epilogue buffers (NQ = 2)");
static_assert(at_epilogue_bytes<4>() <= AtLayout<4>::kMiscOff, "epilogue buffers (NQ = 4)");
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

// Byte offset of 16-byte unit u (0..3) of row r inside a 64B-swizzled
// [rows][64 B] block (the 16-byte unit index XOR bits 1-2 of the row).
__device__ __forceinline__ uint32_t swz64(int r, int u) {
  return (uint32_t)(r * 64 + ((u ^ ((r >> 1) & 3)) << 4));
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

  // the splits of one (token, part) are consecutive in x: one cluster
  const int S = a.splits;
  const int split = blockIdx.x % S;
  const int part = blockIdx.x / S;
  const int row_q = blockIdx.y;  // b * Tq + tq
  const int b = row_q / a.Tq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rope0 = kAtDim - a.rope_dim;
  // 128-dim chunks in streaming order: the others first, then the own ones
  // (own chunks: dims part * kOCols ..).  Closed forms rather than small
  // arrays: a run-time index would put them in local memory, and the MMA
  // operands built from them would no longer be known to be warp-uniform.
  const int own0 = part * kOwn;
  auto chunk_of = [&](int ck) {
    return ck < 4 - kOwn ? (ck < own0 ? ck : ck + kOwn) : own0 + ck - (4 - kOwn);
  };
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
  griddep_wait();  // the predecessor's writes (the selected indices) are visible
  griddep_launch_dependents();
  const int t = a.q_pos[row_q];

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
#pragma unroll 1
      for (int k = 0; k < kMaxK; ++k) {  // rolled: runs once per CTA (code size)
        if (k * 128 >= a.topk) break;
        int j = jv[0];
#pragma unroll
        for (int kk = 1; kk < kMaxK; ++kk) j = k == kk ? jv[kk] : j;
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

  // Epilogue helpers (warps 0-3, one head per thread).  The output leaves
  // as 32-dim slabs: bf16 TMA boxes of [128 heads][64 B], 64B-swizzled,
  // staged in shared memory that is idle by then.
  float m_run = -INFINITY, l_run = 0.f;  // this split's softmax state of the thread's head
  bool epi_ok = false;
  auto out_slab = [&](uint8_t* obuf, int sl, int box, float (&o)[32]) {
    const int hd = threadIdx.x;
    const int d0 = part * kOCols + sl * 32;
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
    uint8_t* bx = obuf + box * kAtOutBoxBytes;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<uint4*>(bx + swz64(hd, u)) =
          make_uint4(pack_bf16x2(o[8 * u], o[8 * u + 1]), pack_bf16x2(o[8 * u + 2], o[8 * u + 3]),
                     pack_bf16x2(o[8 * u + 4], o[8 * u + 5]), pack_bf16x2(o[8 * u + 6], o[8 * u + 7]));
  };
  auto store_out = [&](uint8_t* obuf, int sl0, int n) {
    fence_proxy_async_shared();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 0) {
      for (int i = 0; i < n; ++i)
        tma_store_2d(&tm_out, obuf + i * kAtOutBoxBytes, part * kOCols + (sl0 + i) * 32,
                     row_q * kAtHeads);
      bulk_commit();
      bulk_wait_read_all();
    }
  };
  // this CTA's O, slab sl, times w (zero without tiles)
  auto own_slab = [&](int sl, uint32_t lane_base, float w, float (&o)[32]) {
    uint32_t r[32];
    if (ntile > 0) {
      tmem_ld32(t_o + lane_base + (uint32_t)(sl * 32), r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __fmul_rn(__uint_as_float(r[e]), w);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0.f;
    }
  };
  constexpr int kSlabs = kOCols / 32;

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
    for (int i = 0; i < ntile && ok; ++i) {
      const int sb = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], ph, abortp));
      if (!ok) break;
      tc_fence_after();
      const int g0 = r_lo + i * kAtTile;  // list index of row 0 of the tile
      float z[64];  // raw logits q.k (scaled to the log2 domain below)
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(t_s + lane_base + (uint32_t)(sb * 64), ra);
        tmem_ld32(t_s + lane_base + (uint32_t)(sb * 64 + 32), rb);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          z[e] = __uint_as_float(ra[e]);
          z[32 + e] = __uint_as_float(rb[e]);
        }
      }
      // rows of the tile outside the split, padding between the selected and
      // the window rows, and padding at the end are masked; most tiles have
      // none
      const int g1 = g0 + kAtTile - 1;
      if (!(g1 < r_hi && (g1 < n_sel || (g0 >= ps && g1 < pe)))) {
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const int g = g0 + e;
          const bool valid = g < r_hi && (g < n_sel || (g >= ps && g < pe));
          if (!valid) z[e] = -INFINITY;
        }
      }
      float zmax = -INFINITY;
#pragma unroll
      for (int e = 0; e < 64; ++e) zmax = fmaxf(zmax, z[e]);
      const float mt = zmax * a.scale_log2;  // the scale is positive: max commutes
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
      const float neg_m = -m_run;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = ex2_approx(fmaf(z[2 * e], a.scale_log2, neg_m));
        const float p1 = ex2_approx(fmaf(z[2 * e + 1], a.scale_log2, neg_m));
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
      if (S == 1) {
        // shared memory is idle once the last PV has landed
        const float sink_l2 = a.sink[head] * 1.4426950408889634f;
        const float mm = fmaxf(m_run, sink_l2);
        const float den = (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - mm)) +
                          exp2f(sink_l2 - mm);
        const float scl =
            (m_run == -INFINITY || !(den > 0.f)) ? 0.f : exp2f(m_run - mm) / den;
#pragma unroll 1
        for (int sl = 0; sl < kSlabs; ++sl) {
          float o[32];
          own_slab(sl, lane_base, scl, o);
          out_slab(base_ptr, sl, sl, o);
        }
        store_out(base_ptr, 0, kSlabs);
      } else {
        // split-KV: publish this split's (m, l) and the slabs of O that the
        // other splits of the cluster merge (layout per unit: [slab][16-byte
        // unit u][head][4 floats], so that a warp's stores coalesce)
        const size_t unit = ((size_t)row_q * NQ + part) * S + split;
        float* pml = a.part_ml + unit * 2 * kAtHeads;
        pml[head] = m_run;
        pml[kAtHeads + head] = l_run;
        float* dst = a.part_o + unit * kAtHeads * kOCols;
        const int my_lo = split * kSlabs / S, my_hi = (split + 1) * kSlabs / S;
#pragma unroll 1
        for (int sl = 0; sl < kSlabs; ++sl) {
          if (sl >= my_lo && sl < my_hi) continue;
          float o[32];
          own_slab(sl, lane_base, 1.f, o);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4*>(dst + ((size_t)(sl * 8 + u) * kAtHeads + head) * 4) =
                make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
      }
    }
    epi_ok = ok;
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
        const int chunk = chunk_of(ck);
        const int slot = n % kSlots;
        okp = mbar_wait(&sm.empty[slot], ((uint32_t)(n / kSlots) & 1u) ^ 1u, abortp);
        if (okp && !staged && slot >= kSlots - Lay::kQStage) {  // slot still holds q staging
          okp = mbar_wait(&sm.q_ready, 0, abortp);
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
    // ring slot of own chunk oc of tile j: chunk n = 4 j + ck goes to slot
    // n % kSlots, and the own chunks are the last kOwn of a tile
    auto own_slot = [&](int j, int oc) { return (4 * j + (4 - kOwn) + oc) % kSlots; };
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
            sw128_desc(smem_u32(ring + own_slot(j, oc) * kAtChunkBytes), kAtChunkBytes / 2, 1024);
#pragma unroll
        for (int ks = 0; ks < kAtTile / 16; ++ks)
          mma_ts(t_o + (uint32_t)(oc * 128), t_s + (uint32_t)(sb * 64 + ks * 8),
                 vd0 + (uint64_t)((ks * 16 * 128) >> 4), id_pv, (j > 0 || ks > 0) ? 1u : 0u);
      }
#pragma unroll
      for (int oc = 0; oc < kOwn; ++oc) tc_commit(&sm.empty[own_slot(j, oc)]);
      tc_commit(&sm.pv_done[sb]);
      last_pv = j;
      return true;
    };
    int pv_next = 0;  // next tile whose PV is still to be issued
    for (int i = 0; i < ntile && okm; ++i) {
      const int sb = i & 1;
      if (i >= 2 && pv_next <= i - 2) {
        // P(i-2) lives in S[sb]: its PV is issued before S(i) overwrites it.
        // MMAs of one thread execute in issue order, so the PV reads P before
        // the QK MMAs below write that TMEM; no wait for its completion.
        okm = issue_pv(pv_next++);
        if (!okm) break;
      }
      // S(i) = Q K_i^T over the four 128-dim chunks (others first)
      for (int ck = 0; ck < 4 && okm; ++ck, ++n) {
        const int chunk = chunk_of(ck);
        const bool own = ck >= 4 - kOwn;
        const int slot = n % kSlots;
        // wait for the chunk; meanwhile the previous tile's PV goes in as
        // soon as its P is ready (so that its V slots are released early)
        {
          const uint32_t fph = (uint32_t)(n / kSlots) & 1u;
          if (!mbar_try_wait(&sm.full[slot], fph)) {
            const uint64_t t_start = globaltimer();
            for (uint32_t it = 1;; ++it) {
              if (pv_next == i - 1 &&
                  mbar_try_wait(&sm.p_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u)) {
                okm = issue_pv(pv_next++);
                if (!okm) break;
              }
              if (mbar_try_wait(&sm.full[slot], fph)) break;
              if ((it & 63u) == 0u) {
                if (*abortp) {
                  okm = false;
                  break;
                }
                if (globaltimer() - t_start > kWaitLimitNs) {
                  *abortp = 1;
                  report_error(CSA_ERR_DEVICE_TIMEOUT);
                  okm = false;
                  break;
                }
              }
            }
          }
        }
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
  if (S > 1) {
    // ======================= split-KV merge inside the cluster: after the
    // barrier every split's (m, l) and partial O are visible; CTA `split`
    // merges output slabs [split * kSlabs / S, (split + 1) * kSlabs / S) in
    // split order (its own O straight from TMEM, the others' from a bulk
    // copy).  Products and sums are rounded one by one, in split order, so
    // the result does not depend on the merging CTA.
    __syncwarp();
    cluster_sync_all();
    if (warp < 4 && epi_ok) {
      const int head = threadIdx.x;
      const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
      const int s_lo = split * kSlabs / S, s_hi = (split + 1) * kSlabs / S, ns = s_hi - s_lo;
      const size_t unit0 = ((size_t)row_q * NQ + part) * S;  // unit of split sp: unit0 + sp
      uint8_t* pbuf = base_ptr;                           // (S - 1) x ns slabs of 16 KB
      uint8_t* obuf = base_ptr + (S - 1) * ns * kAtSlabBytes;  // ns output boxes
      bool okm = ns > 0;
      if (okm && threadIdx.x == 0) {
        fence_proxy_async_global();  // partials written by generic stores, read by bulk copies
        mbar_arrive_expect_tx(&sm.merge_bar, (uint32_t)((S - 1) * ns * kAtSlabBytes));
        for (int sp = 0, j = 0; sp < S; ++sp) {
          if (sp == split) continue;
          bulk_load(pbuf + j * ns * kAtSlabBytes,
                    a.part_o + (unit0 + sp) * kAtHeads * kOCols + (size_t)s_lo * (kAtSlabBytes / 4),
                    (uint32_t)(ns * kAtSlabBytes), &sm.merge_bar);
          ++j;
        }
      }
      // merge weights of the thread's head: exp(m_s - M) / L with the sink
      const float sink_l2 = a.sink[head] * 1.4426950408889634f;
      float mv[kAtMaxSplits], lv[kAtMaxSplits];
#pragma unroll
      for (int sp = 0; sp < kAtMaxSplits; ++sp) {
        mv[sp] = -INFINITY;
        lv[sp] = 0.f;
        if (sp < S) {
          const float* ml = a.part_ml + (unit0 + sp) * 2 * kAtHeads;
          mv[sp] = sp == split ? m_run : __ldcg(ml + head);
          lv[sp] = sp == split ? l_run : __ldcg(ml + kAtHeads + head);
        }
      }
      float M = sink_l2;
#pragma unroll
      for (int sp = 0; sp < kAtMaxSplits; ++sp) M = fmaxf(M, mv[sp]);
      float L = exp2f(sink_l2 - M);
#pragma unroll
      for (int sp = 0; sp < kAtMaxSplits; ++sp)
        if (mv[sp] != -INFINITY) L += lv[sp] * exp2f(mv[sp] - M);
      const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
      for (int sp = 0; sp < kAtMaxSplits; ++sp)
        mv[sp] = mv[sp] == -INFINITY ? 0.f : exp2f(mv[sp] - M) * inv;  // now the weights
      if (okm) okm = __all_sync(0xffffffffu, mbar_wait(&sm.merge_bar, 0, abortp));
      {  // the four warps agree before the named barrier of store_out
        uint32_t all;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
            "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(all)
            : "r"(okm ? 1u : 0u)
            : "memory");
        okm = all != 0;
      }
      if (okm) {
        // Rolled loops: this code runs once per CTA, so its size (instruction
        // fetch) costs more than loop overhead.  The sum starts at -0, which
        // adds exactly (x + -0 = x), so the first split enters unchanged.
#pragma unroll 1
        for (int sl = s_lo; sl < s_hi; ++sl) {
          float o[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = -0.f;
#pragma unroll 1
          for (int sp = 0, j = 0; sp < S; ++sp) {
            float wsp = mv[0];
#pragma unroll
            for (int k = 1; k < kAtMaxSplits; ++k) wsp = sp == k ? mv[k] : wsp;
            float tm[32];
            if (sp == split) {
              own_slab(sl, lane_base, wsp, tm);
            } else {
              const uint8_t* src = pbuf + (j * ns + (sl - s_lo)) * kAtSlabBytes;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float4 x = *reinterpret_cast<const float4*>(src + (u * kAtHeads + head) * 16);
                tm[4 * u] = __fmul_rn(x.x, wsp);
                tm[4 * u + 1] = __fmul_rn(x.y, wsp);
                tm[4 * u + 2] = __fmul_rn(x.z, wsp);
                tm[4 * u + 3] = __fmul_rn(x.w, wsp);
              }
              ++j;
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __fadd_rn(o[e], tm[e]);
          }
          out_slab(obuf, sl, sl - s_lo, o);
        }
        store_out(obuf, s_lo, ns);
      }
    }
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
