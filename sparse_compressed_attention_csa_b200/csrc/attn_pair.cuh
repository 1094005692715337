// Steps 3 and 4 on tensor cores, for the measured shape (128 query heads x
// 512 dims, bf16): shared-KV MQA over the selected compressed entries (CSA)
// or every visible entry (HCA), plus the raw window, with the per-head sink
// and partial RoPE ("Compressed Sparse Attention", "Heavily Compressed
// Attention", "Partial RoPE" and "Output gate + sink" rows).
//
// One query token = one MMA M of 128 heads.  Its output O (128 x 512 fp32)
// alone would fill all of TMEM, so a token is served by a PAIR of CTAs (two
// ranks of one thread-block cluster), each owning half of the 512 dims for
// both products:
//
//   S_c = Q[:, D_c] K[:, D_c]^T        partial logits over the CTA's 256 dims
//   S   = S_0 + S_1                    the pair swaps S_c through distributed
//                                      shared memory (fp16, scaled to log2)
//   O[:, D_c] += P V[:, D_c]           P = online softmax of S
//
// so every KV row is gathered once (each CTA reads its own 512 bytes of it)
// and Q K^T is computed once.  TMEM per CTA: O [0,256) | S0 [256,320) |
// S1 [320,384) | Q[:, D_c] as bf16 pairs [384,512).  Shared memory: a ring
// of 10 chunks of 64 rows x 128 dims (a tile's two chunks sit in adjacent
// slots, so one N = 256 MMA covers the tile's PV), three 16 KB receive
// buffers for the partner's partial logits, the row list.  Distributed
// shared memory moves only ~14 GB/s per SM each way (measured with
// st.async; ~20 with bulk copies), so the 16 KB of a tile take ~1.1 us.
//
//   warp 8 (one thread): MMAs   S(i) = Q K_i^T (N = 64, K = 256, A from TMEM)
//                               O   += P(j) V(j) (N = 256, A = P from TMEM)
//   warps 4-7: q by TMA, the row list (the window's rows first: their
//              leading tiles are gathered while the selection's indices
//              load), then the gather: 16-byte cp.async of the CTA's half
//              of each row into 128B-swizzled chunks (FP8 codes: TMA
//              tile::gather4); warp 4 + (2 (i % 2) + c) fetches chunk c of
//              tile i.
//   warps 0-3: one head per thread (= TMEM lane): this CTA's partial logits
//              of each tile, rounded to fp16, out to the partner (st.async
//              into its receive buffers), the partner's in; online softmax
//              in the log2 domain with a lazy rescale, P back into TMEM as
//              bf16; epilogue with the sink, the inverse output rotation
//              and a TMA store.
//
// The pair swaps the scaled partial logits rounded to fp16; each CTA adds
// its own fp32 partial to the partner's fp16 one (one rounding of 2^-11
// relative on half of each logit; beyond +-65504 in log2 units the partial
// saturates).  The two CTAs of a pair may therefore take slightly different
// softmax weights; each normalises its own half of O with its own sums.
//
// Split-KV (few query tokens): the S splits of a token are further pairs
// (grid x = 2 * split + part).  Each CTA of a split writes its unnormalised
// O and its (m, l) to the workspace through shared memory and bulk copies;
// k_attn_merge, launched right after, combines the splits.
//
// FP8 KV cache (kFp8): the caches hold E4M3 codes with one fp32 scale per
// row (quantized after RoPE).  Two gather warps land each chunk's codes (64
// rows x 128 B) in the upper half of its ring slot and its row scales in
// shared memory; two expanding warps rewrite each row in place as bf16
// (code value x row scale, rounded once) in the slot's 128B-swizzled layout
// and release the slot to the MMA.  The rest of the kernel is the bf16 one.
//
// Every mbarrier wait is bounded (a.wait_ns); a wait that runs out records
// CSA_ERR_DEVICE_TIMEOUT and the CTA winds down: it drains every copy and
// MMA it issued and every partner store it expects, reaches every cluster
// barrier, frees TMEM and exits.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kApHeads = 128;
constexpr int kApDim = 512;
constexpr int kApHalf = 256;                         // dims per CTA of the pair
constexpr int kApTile = 64;                          // KV rows per tile (QK N)
constexpr int kApChunkBytes = kApTile * 128 * 2;     // 64 rows x 128 dims bf16
constexpr int kApSlots = 10;                         // ring: 5 tiles of 2 chunks
constexpr int kApQSlot0 = kApSlots - 4;              // q staging: the last 4 slots
constexpr int kApXBytes = kApHeads * kApTile * 2;    // fp16 partial logits of a tile
constexpr int kApXBufs = 3;                          // receive buffers (see the exchange)
constexpr int kApSubBytes = kApHeads * 128;          // q box: [128 heads][64 dims]
constexpr int kApRowCap = 2048;                      // rows per query token
constexpr int kApMaxRope = 128;                      // rotated dims supported
constexpr int kApMaxSplits = 8;                      // split-KV parts per query token
constexpr int kApSlabBytes = kApHeads * 32 * 2;      // 32 dims of fp16 O, 128 heads
constexpr int kApOutBoxBytes = kApHeads * 64;        // 32 dims of bf16 output, 128 heads
constexpr int kApSlabs = kApHalf / 32;
constexpr int kApThreads = 288;      // 9 warps
constexpr int kApThreadsFp8 = 352;   // FP8 caches: 2 more expanding warps (9, 10)
constexpr float kApRescaleLog2 = 8.0f;
constexpr int kApXOff = kApSlots * kApChunkBytes;
constexpr int kApMiscOff = kApXOff + kApXBufs * kApXBytes;
constexpr uint64_t kApDrainNs = 100000000ull;        // 100 ms for the wind-down waits

struct AttnPairArgs {
  const __nv_bfloat16* q;
  const int* q_pos;
  const __nv_bfloat16* kv_cmp;
  const int* idx;    // CSA
  const int* n_cmp;  // HCA
  int n_max;
  const __nv_bfloat16* kv_raw;
  const float* cmp_scale;  // FP8 caches: [B * n_max] and [B * raw_max] row scales
  const float* raw_scale;
  const int* raw_pos0;
  const int* n_raw;
  int raw_max;
  const float* sink;
  int Tq, topk, window, width, stride, rope_dim;
  int rows_per_layer;  // B * Tq: grid row y is layer y / rows_per_layer (own q, sink, out)
                       // of token y % rows_per_layer (shared entries, selection, window)
  float scale_log2;
  int splits;
  unsigned long long wait_ns;  // limit of every bounded wait
  __nv_bfloat16* out;          // splits == 1
  __half* part_o;  // splits > 1: [B*Tq][splits][2][8 slabs][4 units][128][8] O / l, fp16
  float* part_ml;  // [B*Tq][splits][2][2][128]  (m, l) in the log2 domain
  double freq[kApMaxRope / 2];  // RoPE frequencies theta^(-2i/rope_dim)
};

struct ApMisc {
  int rows[kApRowCap];  // gather row coordinates
  float cs[kApMaxRope / 2], sn[kApMaxRope / 2];
  uint64_t full[kApSlots], empty[kApSlots];
  uint64_t stage[kApSlots];  // FP8: a chunk's codes have landed in its slot
  float scl[kApSlots][kApTile];  // FP8: the row scales of each slot's chunk
  uint64_t s_full[2], p_full[2], pv_done[2], xfull[kApXBufs];
  uint64_t q_tma, q_ready, rows_ready, rope_ready, mma_drain;
  uint32_t tmem_base;
  int n_rows;  // padded rows (multiple of 4)
  int n_win;   // window rows (valid rows [0, n_win))
  int n_sel;   // selected / visible entries (valid rows [pad4(n_win), pad4(n_win) + n_sel))
  int abort_flag;
  int scan_tmp[4];
  int last_n[kApSlots];  // last chunk requested into each ring slot (-1: none)
};

constexpr size_t kApSmemBytes = (size_t)kApMiscOff + sizeof(ApMisc) + 1024;
static_assert(kApSmemBytes <= 232448, "shared memory budget");

// The epilogue stages the output in the idle ring: 8 bf16 boxes of 8 KB
// (one split), or the 8 fp16 slabs of 8 KB of the split's O / l (splits).
static_assert(kApSlabs * kApSlabBytes <= kApXOff, "epilogue staging fits the ring");

// 2^x by the hardware approximation (relative error ~2^-22; the softmax
// weights are rounded to bf16 right after).
__device__ __forceinline__ float ap_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t ap_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two floats to fp16 pairs, round to nearest, saturating at +-65504.
__device__ __forceinline__ uint32_t ap_f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float2 ap_f16x2_to_f32(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// Byte offset of 16-byte unit u (0..7) of row r inside a 128B-swizzled
// [rows][128 B] block (atoms of 8 rows).
__device__ __forceinline__ uint32_t ap_swz(int r, int u) {
  return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
}

// Byte offset of 16-byte unit u (0..3) of row r inside a 64B-swizzled
// [rows][64 B] block (the 16-byte unit index XOR bits 1-2 of the row).
__device__ __forceinline__ uint32_t ap_swz64(int r, int u) {
  return (uint32_t)(r * 64 + ((u ^ ((r >> 1) & 3)) << 4));
}

// FP8 caches: expand row r of a chunk from its E4M3 codes (128 B at the
// upper half of the slot, row-major) to bf16 (code value x scale, rounded
// once): dims 0-63 into the lower half, 64-127 into the upper half over the
// row's own codes, both in the 128B-swizzled layout the MMA reads.  The
// thread loads all of the row's codes before it writes any byte.
__device__ __forceinline__ void ap_expand_fp8_row(uint8_t* slot, int r, float scale) {
  const uint4* src = reinterpret_cast<const uint4*>(slot + kApChunkBytes / 2 + r * 128);
  uint4 c[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) c[u] = src[u];
#pragma unroll
  for (int u = 0; u < 8; ++u) {  // codes 16u .. 16u + 15
    const uint32_t w[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {  // codes 4k + 2hw, 4k + 2hw + 1
        const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(
            (__nv_fp8x2_storage_t)((w[k] >> (16 * hw)) & 0xFFFFu), __NV_E4M3);
        const float2 f = __half22float2(__half2(h2));
        o[2 * k + hw] = ap_bf16x2(f.x * scale, f.y * scale);
      }
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {  // bf16 unit 2u + v of the row (8 dims)
      const int unit = 2 * u + v, hh = unit >> 3, uu = unit & 7;
      *reinterpret_cast<uint4*>(slot + hh * (kApChunkBytes / 2) + r * 128 + ((uu ^ (r & 7)) << 4)) =
          make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
    }
  }
}

// Zero row r of a chunk (both halves): masked rows past the split's end.
__device__ __forceinline__ void ap_zero_row(uint8_t* slot, int r) {
#pragma unroll
  for (int unit = 0; unit < 16; ++unit)
    *reinterpret_cast<uint4*>(slot + (unit >> 3) * (kApChunkBytes / 2) + r * 128 +
                              ((unit & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
}

// All 128 threads of warps 0-3 agree on `ok` (named barrier 1).
__device__ __forceinline__ bool ap_softmax_all(bool ok) {
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(all)
      : "r"(ok ? 1u : 0u)
      : "memory");
  return all != 0;
}

template <bool kHca, bool kFp8>
__global__ void __launch_bounds__(kFp8 ? kApThreadsFp8 : kApThreads, 1)
    k_attn_pair(AttnPairArgs a, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_out,
                const __grid_constant__ CUtensorMap tm_cmp,
                const __grid_constant__ CUtensorMap tm_raw) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base_ptr = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
  uint8_t* ring = base_ptr;                // kApSlots x 16 KB
  uint8_t* xbuf = base_ptr + kApXOff;      // kApXBufs x 16 KB: the partner's partial logits
  uint8_t* q_stage = ring + kApQSlot0 * kApChunkBytes;
  ApMisc& sm = *reinterpret_cast<ApMisc*>(base_ptr + kApMiscOff);

  const int S = a.splits;
  const uint32_t rank = cluster_ctarank();  // the cluster is the pair: x = 2 * split + part
  const uint32_t peer = rank ^ 1u;
  const int part = (int)rank;
  const int split = (int)(blockIdx.x >> 1);
  const int row_all = blockIdx.y;               // layer * B * Tq + b * Tq + tq
  const int row_q = row_all % a.rows_per_layer;  // b * Tq + tq: entries, selection, window
  const int layer = row_all / a.rows_per_layer;  // q, sink and out of this layer
  const int b = row_q / a.Tq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rope0 = kApDim - a.rope_dim;
  const int dim0 = part * kApHalf;  // first of the CTA's dims
  const uint64_t wait_ns = a.wait_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kApSlots; ++s) {
      // bf16: the 32 lanes of the gathering warp (cp.async arrivals); FP8: the 2 expanders
      mbar_init(&sm.full[s], kFp8 ? 2 : 32);
      mbar_init(&sm.empty[s], 1);
      mbar_init(&sm.stage[s], 1);  // FP8: expect_tx + the codes' bytes
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.pv_done[i], 1);
    }
    for (int i = 0; i < kApSlots; ++i) sm.last_n[i] = -1;
    for (int i = 0; i < kApXBufs; ++i) mbar_init(&sm.xfull[i], 1);  // expect_tx + 16 KB in
    mbar_init(&sm.q_tma, 1);
    mbar_init(&sm.q_ready, 128);
    mbar_init(&sm.rows_ready, 128);
    mbar_init(&sm.rope_ready, 32);
    mbar_init(&sm.mma_drain, 1);
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
  // the partner's barriers are initialised before any remote access
  __syncwarp();
  cluster_sync_all();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t t_o = tmem, t_s = tmem + 256, t_q = tmem + 384;
  volatile int* abortp = &sm.abort_flag;
  griddep_wait();  // the predecessor's writes (the selected indices) are visible
  griddep_launch_dependents();
  const int t = a.q_pos[row_q];

  if (warp == 4 && lane == 0) {
    // q[:, D_c] of this token: 4 boxes of [128 heads][64 dims], 128B swizzle
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_out);
    tma_prefetch_desc(&tm_cmp);
    tma_prefetch_desc(&tm_raw);
    mbar_arrive_expect_tx(&sm.q_tma, kApHeads * kApHalf * 2);
    for (int sb = 0; sb < 4; ++sb)
      tma_load_2d(q_stage + sb * kApSubBytes, &tm_q, &sm.q_tma, dim0 + sb * 64,
                  row_all * kApHeads);
  }
  if (warp == 8) {
    // RoPE table at the query position
    for (int i = lane; i < a.rope_dim / 2; i += 32) {
      float c, s;
      rope_cs_reduced(t, a.freq[i], &c, &s);
      sm.cs[i] = c;
      sm.sn[i] = s;
    }
    mbar_arrive(&sm.rope_ready);
  }

  // The row list: the window's raw rows (padded to a multiple of 4), then
  // the selected (or, for HCA, every visible) entries in their order (padded
  // likewise).  Global tile t (64 rows of the list) belongs to split t % S:
  // this CTA's tile i is global tile split + i * S, so the window's tiles,
  // known without the selection, lead the first splits.
  auto tile_row0 = [&](int i) { return (split + i * S) * kApTile; };

  // One chunk's gathers (the slot is free), bf16 rows: 16-byte cp.async, lane
  // l copies unit l % 8 of rows 4k + l / 8 (k = 0..15), both 64-dim halves,
  // into the 128B-swizzled layout (a warp instruction reads four whole
  // 128-byte row segments); rows at or past n_rows are zero-filled, so that
  // masked rows hold finite values.  Each lane arrives on the slot's full
  // barrier when its copies have landed (32 arrivals).
  auto gather_chunk_bf16 = [&](int i, int ck, int n_rows, int pw) {
    const int n = 2 * i + ck;
    const int slot = n % kApSlots;
    const uint32_t cbase = smem_u32(ring + slot * kApChunkBytes);
    const int g0 = tile_row0(i);
    const int u = lane & 7, rsub = lane >> 3;
    const size_t col = (size_t)(dim0 + ck * 128) * 2 + (size_t)u * 16;  // byte in the row
    if (lane == 0) sm.last_n[slot] = n;
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
      const int r = 4 * k + rsub;  // row of the chunk
      const int g = g0 + r;
      const bool valid = g < n_rows;
      const char* src = reinterpret_cast<const char*>(a.q);  // read only when valid
      if (valid)
        src = reinterpret_cast<const char*>(g < pw ? a.kv_raw : a.kv_cmp) +
              (size_t)sm.rows[g] * (kApDim * 2) + col;
      const uint32_t d0 = cbase + (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
      cp_async16(d0, src, valid);
      cp_async16(d0 + kApChunkBytes / 2, src + 128, valid);
    }
    cp_async_arrive(&sm.full[slot]);
  };
  // FP8: lanes 0-15 each gather the codes of rows 4l .. 4l + 3 (128 B a row)
  // into the upper half of the slot; the rows' scales go to sm.scl.
  auto gather_chunk_fp8 = [&](int i, int ck, int n_rows, int pw) {
    const int n = 2 * i + ck;
    const int slot = n % kApSlots;
    const int g0 = tile_row0(i);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int gi = g0 + lane + 32 * q;
      sm.scl[slot][lane + 32 * q] =
          gi < n_rows ? (gi < pw ? a.raw_scale : a.cmp_scale)[sm.rows[gi]] : 0.f;
    }
    const int g = g0 + 4 * lane;
    const bool gv = lane < 16 && g < n_rows;
    const unsigned vmask = __ballot_sync(0xffffffffu, gv);  // also orders the scales
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.stage[slot], (uint32_t)__popc(vmask) * 512u);
      sm.last_n[slot] = n;
    }
    __syncwarp();
    if (gv)
      tma_gather4(ring + slot * kApChunkBytes + kApChunkBytes / 2 + lane * 512,
                  g < pw ? &tm_raw : &tm_cmp, &sm.stage[slot], dim0 + ck * 128, sm.rows[g],
                  sm.rows[g + 1], sm.rows[g + 2], sm.rows[g + 3]);
  };

  int early = 0;  // warps 4-7: this CTA's leading tiles already gathered from the window
  if (warp >= 4 && warp < 8) {
    // ======================= row list (warps 4-7); both CTAs of a pair
    // build the same list.  CSA: the selection's entries are loaded first;
    // the window part is written and its leading tiles gathered while the
    // loads are in flight, then the selection is placed after it.
    const int tid = threadIdx.x - 128;
    const int cmp_y0 = b * a.n_max;
    const int raw_y0 = b * a.raw_max;
    constexpr int kMaxE = kApRowCap / 128;
    int jv[kMaxE];
    const int E = kHca ? 0 : (a.topk + 127) / 128;
    if (!kHca) {
      // thread tid compacts entries [tid * E, tid * E + E) of the selection
      const int* sel = a.idx + (size_t)row_q * a.topk;
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
        const int i = tid * E + e;
        jv[e] = (e < E && i < a.topk) ? sel[i] : -1;
      }
    }
    const int rp0 = a.raw_pos0[b];
    const int nraw = a.n_raw[b];
    const int w_lo = max(max(0, t - a.window + 1), rp0);
    const int w_hi = min(t, rp0 + min(nraw, a.raw_max) - 1);
    int n_win = (a.window > 0 && w_hi >= w_lo) ? w_hi - w_lo + 1 : 0;
    n_win = max(0, min(n_win, kApRowCap));
    const int pw = (n_win + 3) & ~3;
    for (int u = tid; u < pw; u += 128)
      sm.rows[u] = raw_y0 + (w_lo - rp0) + (u < n_win ? u : 0);
    int n_sel = 0;
    if (kHca) {
      n_sel = min(min(n_visible(t, a.n_cmp[b], a.width, a.stride), a.n_max), kApRowCap - pw);
      for (int j = tid; j < n_sel; j += 128) sm.rows[pw + j] = cmp_y0 + j;
    } else {
      asm volatile("bar.sync 2, 128;" ::: "memory");  // window rows written
      // leading tiles of window rows only, gathered before the selection is
      // placed: at most 3, whose chunks take ring slots 0-5 for the first
      // time (no wait on a slot or on the q staging)
      while (early < 3 && tile_row0(early) + kApTile <= pw) ++early;
      if (kFp8) {
        if (warp < 6)
          for (int i = 0; i < early; ++i) gather_chunk_fp8(i, warp - 4, pw, pw);
      } else {
        for (int i = (warp - 4) >> 1; i < early; i += 2) gather_chunk_bf16(i, (warp - 4) & 1, pw, pw);
      }
      // the selection: one block scan of the valid counts places it
      int cnt = 0;
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
        if (jv[e] >= a.n_max) {
          report_error(CSA_ERR_DEVICE_BOUNDS);
          jv[e] = -1;
        }
        cnt += jv[e] >= 0 ? 1 : 0;
      }
      int x = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += n;
      }
      if (lane == 31) sm.scan_tmp[warp - 4] = x;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      int off = x - cnt, tot = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int c = sm.scan_tmp[w];
        off += w < warp - 4 ? c : 0;
        tot += c;
      }
      const int cap = kApRowCap - pw;
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
        if (jv[e] >= 0) {
          if (off < cap) sm.rows[pw + off] = cmp_y0 + jv[e];
          ++off;
        }
      }
      n_sel = min(tot, cap);
    }
    const int ps = (n_sel + 3) & ~3;
    for (int k = n_sel + tid; k < ps; k += 128) sm.rows[pw + k] = cmp_y0;  // masked padding
    if (tid == 0) {
      sm.n_sel = n_sel;
      sm.n_win = n_win;
      sm.n_rows = pw + ps;
    }
    asm volatile("bar.sync 2, 128;" ::: "memory");  // rows written
    mbar_arrive(&sm.rows_ready);
  }

  // this split's tiles (each role waits for rows_ready before reading the
  // list); the two CTAs of a pair take the same rows
  bool rows_ok = false;
  int n_rows = 0, ntile = 0;
  auto load_split = [&]() {
    rows_ok = mbar_wait(&sm.rows_ready, 0, abortp, wait_ns);
    n_rows = rows_ok ? sm.n_rows : 0;
    const int tiles = (n_rows + kApTile - 1) / kApTile;
    ntile = tiles > split ? (tiles - split + S - 1) / S : 0;
  };

  // exchange bookkeeping of thread 0: partner tiles whose 16 KB this CTA
  // expects (expect_tx posted) and has received
  int x_posted = 0, x_recv = 0;

  if (warp < 4) {
    // ======================= softmax / exchange / epilogue warps
    const int head = warp * 32 + lane;  // TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;  // this split's softmax state of the head (log2)
    // ---- q: staged boxes to TMEM, RoPE on the rotated dims (bf16 pairs)
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_tma, 0, abortp, wait_ns) &&
                                          mbar_wait(&sm.rope_ready, 0, abortp, wait_ns));
    if (ok) {
#pragma unroll 1
      for (int sb = 0; sb < 4; ++sb) {
        const int d0 = dim0 + sb * 64;
        const uint8_t* blk = q_stage + sb * kApSubBytes;
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = *reinterpret_cast<const uint4*>(blk + ap_swz(head, u));
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        if (d0 + 64 > rope0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int d = d0 + 2 * e;
            if (d >= rope0) {
              const int i = (d - rope0) >> 1;
              __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162*>(&w[e]);
              const float2 f = __bfloat1622float2(h2);
              w[e] = ap_bf16x2(f.x * sm.cs[i] - f.y * sm.sn[i], f.x * sm.sn[i] + f.y * sm.cs[i]);
            }
          }
        }
        uint32_t r16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) r16[e] = w[e];
        tmem_st16(t_q + lane_base + (uint32_t)(sb * 32), r16);
#pragma unroll
        for (int e = 0; e < 16; ++e) r16[e] = w[16 + e];
        tmem_st16(t_q + lane_base + (uint32_t)(sb * 32 + 16), r16);
      }
    }
    tmem_wait_st();
    fence_proxy_async_shared();
    tc_fence_before();
    mbar_arrive(&sm.q_ready);
    load_split();
    ok = ok && __all_sync(0xffffffffu, rows_ok);
    if (threadIdx.x == 0) {  // the partner's first tiles
      x_posted = min(ntile, kApXBufs);
      for (int i = 0; i < x_posted; ++i) mbar_arrive_expect_tx(&sm.xfull[i], kApXBytes);
    }
    const uint32_t peer_x = mapa(xbuf, peer);  // the partner's receive buffers
    const uint32_t peer_xfull = mapa(&sm.xfull[0], peer);
    const uint32_t xrow = (uint32_t)head * 128u;

    // ---- online softmax over the tiles
    // Exchange: tile i's partial logits go to the partner's buffer i % 3.
    // Three buffers need no handshake: before this CTA can send tile i + 3,
    // its QK(i + 3) needs the PV of tile i + 1 issued, hence P(i + 1), hence
    // the partner's tile i + 1, which the partner sends only after it has
    // read tile i from that buffer (each thread reads tile i before it sends
    // tile i + 1).  (Sending one tile ahead of the softmax instead measured
    // slower: with two S buffers the next QK is not ready in time.)
    // valid rows: the window's [0, n_win) and the entries' [pw, pe)
    const int nw = sm.n_win, pw = (nw + 3) & ~3, pe = pw + sm.n_sel;
    for (int i = 0; i < ntile && ok; ++i) {
      const int sb = i & 1;
      const int xb = i % kApXBufs;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&sm.s_full[sb], (uint32_t)(i >> 1) & 1u, abortp, wait_ns));
      if (!ok) break;
      tc_fence_after();
      // this CTA's partial logits, scaled to the log2 domain (exact fp32)
      float z[64];
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(t_s + lane_base + (uint32_t)(sb * 64), ra);
        tmem_ld32(t_s + lane_base + (uint32_t)(sb * 64 + 32), rb);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          z[e] = __uint_as_float(ra[e]) * a.scale_log2;
          z[32 + e] = __uint_as_float(rb[e]) * a.scale_log2;
        }
      }
      // ---- out: fp16 pairs into the partner's buffer xb
      {
        const uint32_t dst = peer_x + (uint32_t)(xb * kApXBytes) + xrow;
        const uint32_t bar = peer_xfull + (uint32_t)(xb * 8);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = make_uint4(ap_f16x2_sat(z[8 * u], z[8 * u + 1]),
                                     ap_f16x2_sat(z[8 * u + 2], z[8 * u + 3]),
                                     ap_f16x2_sat(z[8 * u + 4], z[8 * u + 5]),
                                     ap_f16x2_sat(z[8 * u + 6], z[8 * u + 7]));
          st_async_v4(dst + (uint32_t)((u ^ (head & 7)) << 4), v, bar);
        }
      }
      // ---- in: the partner's tile i
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(&sm.xfull[xb], (uint32_t)(i / kApXBufs) & 1u,
                                                     abortp, wait_ns));
      if (!ok) break;
      if (threadIdx.x == 0) {
        x_recv = i + 1;
        if (i + kApXBufs < ntile) {  // the partner's tile i + 3 lands in this buffer next
          mbar_arrive_expect_tx(&sm.xfull[xb], kApXBytes);
          x_posted = i + kApXBufs + 1;
        }
      }
      {
        const uint8_t* src = xbuf + xb * kApXBytes + xrow;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + ((u ^ (head & 7)) << 4));
          const float2 f0 = ap_f16x2_to_f32(v.x), f1 = ap_f16x2_to_f32(v.y);
          const float2 f2 = ap_f16x2_to_f32(v.z), f3 = ap_f16x2_to_f32(v.w);
          z[8 * u] += f0.x;
          z[8 * u + 1] += f0.y;
          z[8 * u + 2] += f1.x;
          z[8 * u + 3] += f1.y;
          z[8 * u + 4] += f2.x;
          z[8 * u + 5] += f2.y;
          z[8 * u + 6] += f3.x;
          z[8 * u + 7] += f3.y;
        }
      }
      // rows of the tile outside the split, padding between the selected and
      // the window rows, and padding at the end are masked; most tiles have
      // none
      const int g0 = tile_row0(i);  // list index of row 0 of the tile
      const int g1 = g0 + kApTile - 1;
      if (!(g1 < n_rows && (g1 < nw || (g0 >= pw && g1 < pe)))) {
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const int g = g0 + e;
          const bool valid = g < n_rows && (g < nw || (g >= pw && g < pe));
          if (!valid) z[e] = -INFINITY;
        }
      }
      // tile maximum: eight independent chains, then a tree
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = z[k];
#pragma unroll
      for (int e = 8; e < 64; ++e) mx[e & 7] = fmaxf(mx[e & 7], z[e]);
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      // lazy rescale: a head's running maximum moves only when the tile's
      // exceeds it by more than 2^8 (or on its first finite tile).  The
      // decision is per head (lane), but the wait and the TMEM accesses are
      // warp-collective: when any lane of the warp moves, the whole warp
      // takes the branch, the lanes that keep their maximum with alpha = 1.
      const bool move = mt > m_run + kApRescaleLog2 || m_run == -INFINITY;
      const float m_new = move ? mt : m_run;
      if (i > 0 && __any_sync(0xffffffffu, move && m_run != -INFINITY)) {
        // O holds P V of earlier tiles: wait for the last PV, then rescale
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(i - 1) & 1],
                                               (uint32_t)((i - 1) >> 1) & 1u, abortp, wait_ns));
        if (!ok) break;
        tc_fence_after();
        const float alpha = (move && m_run != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < kApHalf; cc += 32) {
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
      m_run = m_new;
      uint32_t pk[32];
      float ps8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ps8[k] = 0.f;
      const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = ap_ex2(z[2 * e] + neg_m);
        const float p1 = ap_ex2(z[2 * e + 1] + neg_m);
        __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
        const float2 back = __bfloat1622float2(pb);
        ps8[e & 7] += back.x + back.y;
        pk[e] = *reinterpret_cast<uint32_t*>(&pb);
      }
      l_run += ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
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
                                             (uint32_t)((ntile - 1) >> 1) & 1u, abortp, wait_ns));
    ok = ap_softmax_all(ok);  // all four softmax warps agree before the named barriers below
    if (ok) {
      // the ring is idle once the last PV has landed
      tc_fence_after();
      if (S == 1) {
        // normalise with the sink, rotate the output's RoPE dims back by -t,
        // bf16, TMA store of 32-dim boxes ([128 heads][64 B], 64B swizzle)
        const float sink_l2 = a.sink[layer * kApHeads + head] * 1.4426950408889634f;
        const float mm = fmaxf(m_run, sink_l2);
        const float den = (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - mm)) +
                          exp2f(sink_l2 - mm);
        const float scl =
            (m_run == -INFINITY || !(den > 0.f)) ? 0.f : exp2f(m_run - mm) / den;
#pragma unroll 1
        for (int sl = 0; sl < kApSlabs; ++sl) {
          float o[32];
          if (ntile > 0) {
            uint32_t r[32];
            tmem_ld32(t_o + lane_base + (uint32_t)(sl * 32), r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(r[e]) * scl;
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
          }
          const int d0 = dim0 + sl * 32;
          if (d0 + 32 > rope0) {
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
          }
          uint8_t* bx = ring + sl * kApOutBoxBytes;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(bx + ap_swz64(head, u)) = make_uint4(
                ap_bf16x2(o[8 * u], o[8 * u + 1]), ap_bf16x2(o[8 * u + 2], o[8 * u + 3]),
                ap_bf16x2(o[8 * u + 4], o[8 * u + 5]), ap_bf16x2(o[8 * u + 6], o[8 * u + 7]));
        }
        fence_proxy_async_shared();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 0) {
          for (int sl = 0; sl < kApSlabs; ++sl)
            tma_store_2d(&tm_out, ring + sl * kApOutBoxBytes, dim0 + sl * 32, row_all * kApHeads);
          bulk_commit();
          bulk_wait_read_all();
        }
      } else {
        // split-KV: this split's (m, l) and its O / l in fp16 for
        // k_attn_merge (values of order one: fp16 keeps 11 bits).  O leaves
        // through the ring as 8 contiguous 8 KB slabs ([16-byte unit u][head]
        // [8 halves] per 32 dims) and one bulk copy.
        const size_t unit = ((size_t)row_all * S + split) * 2 + part;
        float* pml = a.part_ml + unit * 2 * kApHeads;
        pml[head] = m_run;
        pml[kApHeads + head] = l_run;
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
        for (int sl = 0; sl < kApSlabs; ++sl) {
          uint32_t r[32];
          if (ntile > 0) {
            tmem_ld32(t_o + lane_base + (uint32_t)(sl * 32), r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          uint8_t* slab = ring + sl * kApSlabBytes;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t h[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              h[k] = ap_f16x2_sat(__uint_as_float(r[8 * u + 2 * k]) * inv_l,
                                  __uint_as_float(r[8 * u + 2 * k + 1]) * inv_l);
            *reinterpret_cast<uint4*>(slab + (u * kApHeads + head) * 16) =
                make_uint4(h[0], h[1], h[2], h[3]);
          }
        }
        fence_proxy_async_shared();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 0) {
          bulk_store(a.part_o + unit * kApHeads * kApHalf, ring, kApSlabs * kApSlabBytes);
          bulk_commit();
          bulk_wait_read_all();
        }
      }
    }
  } else if (kFp8 && warp != 8) {
    // ======================= FP8 caches: warps 4-5 gather, 6, 7, 9, 10 expand
    // Chunk n = 2i + c of tile i goes to ring slot n % kApSlots.  Warp 4 + c
    // gathers chunk c of every tile: lanes 0-15 each the codes of rows
    // 4l .. 4l + 3 (128 dims, 128 B a row) into the upper half of the slot,
    // and the rows' scales into sm.scl.  Expanding warp e (warps 6, 7, 9,
    // 10 are e = 0..3) takes chunk c = e % 2, rows 32 (e / 2) + lane: waits
    // for the codes, expands its rows to bf16 in place, and arrives on the
    // slot's full barrier (two arrivals release it to the MMA).  The gathers
    // run ahead of the expansion by up to the ring.
    load_split();
    const int ex = warp < 8 ? warp - 6 : warp - 7;  // expander index (warps 6, 7, 9, 10)
    const int ck = warp < 6 ? warp - 4 : ex & 1;
    const int pw = (sm.n_win + 3) & ~3;
    bool okp = __all_sync(0xffffffffu, rows_ok);
    if (warp < 6) {
      bool staged = false;  // q staging slots handed back
      for (int i = early; i < ntile && okp; ++i) {  // the first `early` went out with the list
        const int n = 2 * i + ck;
        const int slot = n % kApSlots;
        if (lane == 0) {
          okp = mbar_wait(&sm.empty[slot], ((uint32_t)(n / kApSlots) & 1u) ^ 1u, abortp, wait_ns);
          if (okp && !staged && slot >= kApQSlot0) {  // slot still holds q staging
            okp = mbar_wait(&sm.q_ready, 0, abortp, wait_ns);
            staged = true;
          }
        }
        okp = __shfl_sync(0xffffffffu, okp ? 1 : 0, 0) != 0;
        if (!okp) break;
        gather_chunk_fp8(i, ck, n_rows, pw);
      }
    } else {
      for (int i = 0; i < ntile && okp; ++i) {
        const int n = 2 * i + ck;
        const int slot = n % kApSlots;
        okp = __all_sync(0xffffffffu, mbar_wait(&sm.stage[slot], (uint32_t)(n / kApSlots) & 1u,
                                                abortp, wait_ns));
        if (!okp) break;
        const int g0 = tile_row0(i);
        uint8_t* sl = ring + slot * kApChunkBytes;
        const int r = 32 * (ex >> 1) + lane;
        if (g0 + r < n_rows)
          ap_expand_fp8_row(sl, r, sm.scl[slot][r]);
        else
          ap_zero_row(sl, r);
        fence_proxy_async_shared();  // read by the MMA (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.full[slot]);
      }
    }
  } else if (warp < 8) {
    // ======================= gather producers (warps 4-7)
    // Chunk n (tile n / 2, dims dim0 + 128 (n % 2)) goes to ring slot
    // n % kApSlots; warp 4 + (2 (i % 2) + c) fetches chunk c of tile i with
    // one gather4 per lane (gather_chunk_bf16).  The first `early` tiles went
    // out with the row list.
    load_split();
    const int ck = (warp - 4) & 1, tpar = (warp - 4) >> 1;
    const int pw = (sm.n_win + 3) & ~3;
    bool okp = __all_sync(0xffffffffu, rows_ok);
    bool staged = false;  // q staging slots handed back
    for (int i = tpar; i < ntile && okp; i += 2) {
      if (i < early) continue;
      const int n = 2 * i + ck;
      const int slot = n % kApSlots;
      if (lane == 0) {
        okp = mbar_wait(&sm.empty[slot], ((uint32_t)(n / kApSlots) & 1u) ^ 1u, abortp, wait_ns);
        if (okp && !staged && slot >= kApQSlot0) {  // slot still holds q staging
          okp = mbar_wait(&sm.q_ready, 0, abortp, wait_ns);
          staged = true;
        }
      }
      okp = __shfl_sync(0xffffffffu, okp ? 1 : 0, 0) != 0;
      if (!okp) break;
      gather_chunk_bf16(i, ck, n_rows, pw);
    }
    cp_async_wait_all();  // every copy into shared memory lands before the CTA may exit
  } else if (warp == 8 && lane == 0) {
    // ======================= MMA issuer
    constexpr uint32_t id_qk = idesc_bf16_f32(128, kApTile);
    constexpr uint32_t id_pv = idesc_bf16_f32(128, kApHalf, 0, 1);
    load_split();
    bool okm = rows_ok && mbar_wait(&sm.q_ready, 0, abortp, wait_ns);
    tc_fence_after();
    // PV of tile j: P(j) in S[j & 1], V = the tile's two chunks in adjacent
    // slots (2j mod 10, +1): one N = 256 MMA per 16 rows
    auto issue_pv = [&](int j) -> bool {
      const int sb = j & 1;
      if (!mbar_wait(&sm.p_full[sb], (uint32_t)(j >> 1) & 1u, abortp, wait_ns)) return false;
      tc_fence_after();
      const int slot0 = (2 * j) % kApSlots;
      const uint64_t vd0 =
          sw128_desc(smem_u32(ring + slot0 * kApChunkBytes), kApChunkBytes / 2, 1024);
#pragma unroll
      for (int ks = 0; ks < kApTile / 16; ++ks)
        mma_ts(t_o, t_s + (uint32_t)(sb * 64 + ks * 8), vd0 + (uint64_t)((ks * 16 * 128) >> 4),
               id_pv, (j > 0 || ks > 0) ? 1u : 0u);
      tc_commit(&sm.empty[slot0]);
      tc_commit(&sm.empty[slot0 + 1]);
      tc_commit(&sm.pv_done[sb]);
      return true;
    };
    int pv_next = 0;  // next tile whose PV is still to be issued
    int n = 0;        // chunks consumed
    for (int i = 0; i < ntile && okm; ++i) {
      const int sb = i & 1;
      if (i >= 2 && pv_next <= i - 2) {
        // P(i-2) lives in S[sb]: its PV is issued before S(i) overwrites it.
        // MMAs of one thread execute in issue order, so the PV reads P before
        // the QK MMAs below write that TMEM; no wait for its completion.
        okm = issue_pv(pv_next++);
        if (!okm) break;
      }
      for (int ck = 0; ck < 2 && okm; ++ck, ++n) {
        const int slot = n % kApSlots;
        // wait for the chunk; meanwhile the previous tile's PV goes in as
        // soon as its P is ready (so that its slots are released early)
        {
          const uint32_t fph = (uint32_t)(n / kApSlots) & 1u;
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
                if (*abortp || timeout_recorded()) {
                  *abortp = 1;
                  okm = false;
                  break;
                }
                if (globaltimer() - t_start > wait_ns) {
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
        if (!kFp8) fence_proxy_async_shared();  // written by cp.async (generic proxy), read by the MMA
        tc_fence_after();
        const uint64_t bd0 = sw128_desc(smem_u32(ring + slot * kApChunkBytes), 16, 1024);
        const uint32_t a0 = t_q + (uint32_t)(ck * 64);  // q dims ck*128.. as bf16 pairs
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(t_s + (uint32_t)(sb * 64), a0 + (uint32_t)((ks >> 2) * 32 + (ks & 3) * 8),
                 bd0 + (uint64_t)(((ks >> 2) * (kApChunkBytes / 2) + (ks & 3) * 32) >> 4), id_qk,
                 (ck | ks) != 0 ? 1u : 0u);
        if (pv_next == i - 1 &&
            mbar_try_wait(&sm.p_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u))
          okm = issue_pv(pv_next++);
      }
      if (!okm) break;
      tc_commit(&sm.s_full[sb]);
    }
    while (okm && pv_next < ntile) okm = issue_pv(pv_next++);
    // TMEM is freed only after every MMA issued here has landed: one commit
    // tracks them all
    tc_commit(&sm.mma_drain);
    mbar_drain(&sm.mma_drain, 0, kApDrainNs);
  }

  // ======================= wind-down
  // Both CTAs of the pair are past their tile loops: every partial-logit
  // store the partner will issue has been issued.  Those this CTA posted for
  // but did not receive (only after an abort) land before it may exit.
  __syncwarp();
  cluster_sync_all();
  if (threadIdx.x == 0) {
    for (int i = x_recv; i < x_posted; ++i)
      mbar_drain_cluster(&sm.xfull[i % kApXBufs], (uint32_t)(i / kApXBufs) & 1u, kApDrainNs);
  }
  if (warp == 4 && lane == 0) {
    // every copy into shared memory lands before the CTA may exit: q, and in
    // each ring slot the last chunk requested into it (an earlier one was
    // consumed before the slot could be refilled)
    mbar_drain(&sm.q_tma, 0, kApDrainNs);
    for (int s = 0; s < kApSlots; ++s) {
      const int n = sm.last_n[s];
      if (n >= 0)
        mbar_drain(kFp8 ? &sm.stage[s] : &sm.full[s], (uint32_t)(n / kApSlots) & 1u, kApDrainNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Split-KV merge: one CTA per (token, part, 32-dim slab), one head per
// thread.  With the splits' (m_s, l_s) and normalised Ô_s = O_s / l_s:
//   M = max(sink, max_s m_s),  L = 2^(sink - M) + sum_s l_s 2^(m_s - M)
//   o = sum_s (l_s 2^(m_s - M) / L) Ô_s   (split order, products and sums
//                                          rounded one by one: deterministic)
// then the RoPE dims rotated back by -t, bf16.
struct AttnMergeArgs {
  const __half* part_o;
  const float* part_ml;
  const float* sink;
  const int* q_pos;
  int splits;
  int rope_dim;
  int rows_per_layer;  // as in AttnPairArgs
  __nv_bfloat16* out;
  double freq[kApMaxRope / 2];
};

__global__ void __launch_bounds__(kApHeads) k_attn_merge(AttnMergeArgs a) {
  __shared__ float cs[16], sn[16];
  sm100::griddep_wait();  // the partials of the attention kernel are visible
  sm100::griddep_launch_dependents();
  const int part = blockIdx.x >> 3, sl = blockIdx.x & 7;
  const int row_all = blockIdx.y;  // layer * rows_per_layer + token
  const int row_q = row_all % a.rows_per_layer, layer = row_all / a.rows_per_layer;
  const int head = threadIdx.x;
  const int S = a.splits;
  const int rope0 = kApDim - a.rope_dim;
  const int d0 = part * kApHalf + sl * 32;
  const bool rot = d0 + 32 > rope0;
  if (rot && head < 16) {
    const int d = d0 + 2 * head;
    if (d >= rope0) {
      float c, s;
      rope_cs_reduced(a.q_pos[row_q], a.freq[(d - rope0) >> 1], &c, &s);
      cs[head] = c;
      sn[head] = s;
    }
  }
  const size_t unit0 = (size_t)row_all * S * 2 + part;  // unit of split s: unit0 + 2 s
  auto slab_of = [&](int s) {
    return reinterpret_cast<const uint4*>(a.part_o + (unit0 + 2 * (size_t)s) * kApHeads * kApHalf) +
           (size_t)sl * (kApSlabBytes / 16);
  };
  // every split's (m, l) and the first four splits' data, all in flight at once
  float mv[kApMaxSplits], lv[kApMaxSplits];
  uint4 x[4][4];
#pragma unroll
  for (int s = 0; s < kApMaxSplits; ++s) {
    mv[s] = -INFINITY;
    lv[s] = 0.f;
    if (s < S) {
      const float* ml = a.part_ml + (unit0 + 2 * s) * 2 * kApHeads;
      mv[s] = __ldcg(ml + head);
      lv[s] = __ldcg(ml + kApHeads + head);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int u = 0; u < 4; ++u)
      x[j][u] = j < S ? __ldcg(slab_of(j) + u * kApHeads + head) : make_uint4(0u, 0u, 0u, 0u);
  const float sink_l2 = a.sink[layer * kApHeads + head] * 1.4426950408889634f;
  float M = sink_l2;
#pragma unroll
  for (int s = 0; s < kApMaxSplits; ++s) M = fmaxf(M, mv[s]);
  float L = exp2f(sink_l2 - M);
#pragma unroll
  for (int s = 0; s < kApMaxSplits; ++s) {
    mv[s] = mv[s] == -INFINITY ? 0.f : lv[s] * exp2f(mv[s] - M);  // l_s 2^(m_s - M)
    L += mv[s];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  float o[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) o[e] = -0.f;  // x + -0 = x: the first split enters unchanged
  auto accumulate = [&](const uint4 (&v)[4], float w) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t hv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = ap_f16x2_to_f32(hv[k]);
        o[8 * u + 2 * k] = __fadd_rn(o[8 * u + 2 * k], __fmul_rn(f.x, w));
        o[8 * u + 2 * k + 1] = __fadd_rn(o[8 * u + 2 * k + 1], __fmul_rn(f.y, w));
      }
    }
  };
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (j < S) accumulate(x[j], mv[j] * inv);
#pragma unroll
  for (int s0 = 4; s0 < kApMaxSplits; s0 += 4) {
    if (s0 >= S) break;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        x[j][u] = s0 + j < S ? __ldcg(slab_of(s0 + j) + u * kApHeads + head)
                             : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < S) accumulate(x[j], mv[s0 + j] * inv);
  }
  if (rot) {
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int d = d0 + e;
      if (d >= rope0) {  // inverse rotation at -t
        const float x0 = o[e], x1 = o[e + 1];
        o[e] = x0 * cs[e >> 1] + x1 * sn[e >> 1];
        o[e + 1] = -x0 * sn[e >> 1] + x1 * cs[e >> 1];
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(a.out + ((size_t)row_all * kApHeads + head) * kApDim + d0);
#pragma unroll
  for (int u = 0; u < 4; ++u)
    dst[u] = make_uint4(ap_bf16x2(o[8 * u], o[8 * u + 1]), ap_bf16x2(o[8 * u + 2], o[8 * u + 3]),
                        ap_bf16x2(o[8 * u + 4], o[8 * u + 5]), ap_bf16x2(o[8 * u + 6], o[8 * u + 7]));
}

}  // namespace csa
