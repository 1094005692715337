// Step 2b, fast path: exact top-k ("keeps the top 1,024 entries") of one
// query row held in registers, ties to the lower index, output ascending.
//
// Each of NT threads holds PT candidates, striped: candidate slot e of thread
// t is position e * NT + t of the block's range, so the loads coalesce.
// Radix select on order-preserving uint32 keys, 8 bits per pass, starting at
// the highest bit in which the row's keys differ, and stopping as soon as
// the bin that holds the k-th key is taken whole.  Then the kept candidates
// are placed in index order: per (slot, warp) ballots give counts, one
// block scan over those counts (slot-major, then warp) gives each group's
// first output position.
//
// Rows longer than one block's capacity use two stages: each chunk keeps its
// own top-k (k_topk_chunk), then the candidates of all chunks, in index
// order, are selected again (k_topk_merge).  This is exact: an entry in the
// row's top-k is beaten (higher score, or equal score at a lower index) by
// fewer than k entries of the row, hence of its chunk.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

template <int NT, int PT>
struct TopkShared {
  static constexpr int kGroups = PT * (NT / 32);  // (slot, warp) groups in index order
  unsigned hist[256];
  int scan[33];
  uint32_t prefix;
  int remaining;
  int bin_count;
  uint32_t red_and[32], red_or[32];
  int cnt[kGroups];
};

// Exclusive scan, in place, of the kGroups counts in sh.cnt (every thread
// calls it; the counts must have been written before).  Returns the total.
template <int NT, int PT>
__device__ __forceinline__ int scan_groups(TopkShared<NT, PT>& sh) {
  constexpr int G = TopkShared<NT, PT>::kGroups;
  static_assert(G <= NT, "one thread per group");
  __syncthreads();
  const int v = (int)threadIdx.x < G ? sh.cnt[threadIdx.x] : 0;
  int total;
  const int incl = block_inclusive_scan(v, sh.scan, &total);
  if ((int)threadIdx.x < G) sh.cnt[threadIdx.x] = incl - v;
  __syncthreads();
  return total;
}

// Writes index_of(e) of every selected candidate to out[position] (positions
// in index order, only those below k); returns the number selected.
template <int NT, int PT, typename IndexOf>
__device__ __forceinline__ int place_selected(const bool (&sel)[PT], int k, IndexOf index_of,
                                              int* out, TopkShared<NT, PT>& sh) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const unsigned m = __ballot_sync(0xffffffffu, sel[e]);
    if (lane == 0) sh.cnt[e * NW + wid] = __popc(m);
  }
  const int total = scan_groups(sh);
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const unsigned m = __ballot_sync(0xffffffffu, sel[e]);  // recomputed: fewer live registers
    if (sel[e]) {
      const int pos = sh.cnt[e * NW + wid] + __popc(m & lt);
      if (pos < k) out[pos] = index_of(e);
    }
  }
  return total;
}

// Selects the top `k` of the block's candidates.  key[e], valid[e] describe
// candidate slot e (position e * NT + threadIdx.x); index_of(e) gives its
// output index.  Writes the kept indices, ascending, to out[0 .. min(k,
// n_valid)) and returns that count (same value in every thread).
template <int NT, int PT, typename IndexOf>
__device__ int block_topk(const uint32_t (&key)[PT], const bool (&valid)[PT], int k,
                          IndexOf index_of, int* out, TopkShared<NT, PT>& sh) {
  static_assert(NT >= 256, "bin scan needs 256 threads");
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int nv_local = 0;
  uint32_t k_and = 0xffffffffu, k_or = 0u;
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    if (valid[e]) {
      ++nv_local;
      k_and &= key[e];
      k_or |= key[e];
    }
  }
  int n_valid;
  block_inclusive_scan(nv_local, sh.scan, &n_valid);
  if (n_valid <= k) return place_selected<NT, PT>(valid, k, index_of, out, sh);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
    k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
  }
  if (lane == 0) {
    sh.red_and[wid] = k_and;
    sh.red_or[wid] = k_or;
  }
  __syncthreads();
  k_and = 0xffffffffu;
  k_or = 0u;
  for (int w = 0; w < NW; ++w) {
    k_and &= sh.red_and[w];
    k_or |= sh.red_or[w];
  }
  const uint32_t diff = k_and ^ k_or;
  uint32_t prefix, mask;
  int remaining = k;
  if (diff == 0u) {  // all valid keys equal
    prefix = k_and;
    mask = 0xffffffffu;
  } else {
    int hi = 31 - __clz(diff);
    mask = hi == 31 ? 0u : (0xffffffffu << (hi + 1));  // bits above hi are common
    prefix = k_and & mask;
#pragma unroll 1
    while (hi >= 0) {
      const int lo = max(hi - 7, 0);
      const uint32_t dmask = ((hi - lo == 31) ? 0xffffffffu : ((1u << (hi - lo + 1)) - 1u));
      for (int i = threadIdx.x; i < 256; i += NT) sh.hist[i] = 0u;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < PT; ++e)
        if (valid[e] && (key[e] & mask) == prefix)
          atomicAdd(&sh.hist[(key[e] >> lo) & dmask], 1u);
      __syncthreads();
      if (threadIdx.x < 256) {
        // thread b holds bin 255 - b: an inclusive scan gives, per bin, the
        // count of keys in this bin or above
        const int bin = 255 - (int)threadIdx.x;
        const int h = (int)sh.hist[bin];
        int x = h;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += n;
        }
        if (lane == 31) sh.scan[wid] = x;
        asm volatile("bar.sync 3, 256;" ::: "memory");
        int off = 0;
        for (int w = 0; w < wid; ++w) off += sh.scan[w];
        const int incl = off + x, excl = incl - h;
        if (incl >= remaining && excl < remaining) {
          sh.prefix = prefix | ((uint32_t)bin << lo);
          sh.remaining = remaining - excl;
          sh.bin_count = h;
        }
      }
      __syncthreads();
      prefix = sh.prefix;
      remaining = sh.remaining;
      mask |= dmask << lo;
      hi = lo - 1;
      if (remaining == sh.bin_count) break;  // the boundary bin is kept whole
    }
  }
  // Kept: keys above the boundary bin, and the first `remaining` keys (in
  // index order) of the boundary bin.  One scan over the groups, of the
  // greater and equal counts packed in one int (each total < 2^16), places
  // them all: a kept candidate's position is the number of kept ones before
  // it in index order.
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const uint32_t km = key[e] & mask;
    const unsigned mg = __ballot_sync(0xffffffffu, valid[e] && km > prefix);
    const unsigned mq = __ballot_sync(0xffffffffu, valid[e] && km == prefix);
    if (lane == 0) sh.cnt[e * NW + wid] = (__popc(mg) << 16) | __popc(mq);
  }
  scan_groups(sh);
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const uint32_t km = key[e] & mask;
    const bool g = valid[e] && km > prefix, q = valid[e] && km == prefix;
    const unsigned mg = __ballot_sync(0xffffffffu, g);
    const unsigned mq = __ballot_sync(0xffffffffu, q);
    const int before = sh.cnt[e * NW + wid];
    const int g_before = before >> 16, q_before = before & 0xffff;
    const int q_rank = q_before + __popc(mq & lt);  // rank among the boundary keys
    if (g || (q && q_rank < remaining)) {
      // kept before this one: greater ones, plus boundary ones of rank < remaining
      const int pos = g_before + __popc(mg & lt) + min(q_rank, remaining);
      if (pos < k) out[pos] = index_of(e);
    }
  }
  return k;
}

// One CTA per (chunk, query row).  Chunk c covers entries
// [c * NT * PT, (c + 1) * NT * PT) of the row's visible entries.  With one
// chunk per row the result goes to idx_out (padded with -1); otherwise to the
// candidate workspace cand[row][c][k] with its count in cand_n[row][c].
template <int NT, int PT>
__global__ void __launch_bounds__(NT)
    k_topk_chunk(const float* __restrict__ scores, const int* __restrict__ q_pos,
                 const int* __restrict__ n_cmp, int Tq, int n_max, int k, int width, int stride,
                 int n_chunks, int* __restrict__ idx_out, int* __restrict__ cand,
                 int* __restrict__ cand_n) {
  __shared__ TopkShared<NT, PT> sh;
  sm100::griddep_wait();  // the scores of the predecessor are visible
  sm100::griddep_launch_dependents();
  const int c = blockIdx.x, row = blockIdx.y;
  const int b = row / Tq;
  const int base = c * NT * PT + (int)threadIdx.x;
  const float* s = scores + (size_t)row * n_max;
  // the row's scores are loaded up to n_max (in bounds) without waiting for
  // the visible count, then masked
  float v[PT];
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const int j = base + e * NT;
    v[e] = j < n_max ? s[j] : 0.f;
  }
  const int nv = min(n_visible(q_pos[row], n_cmp[b], width, stride), n_max);
  uint32_t key[PT];
  bool valid[PT];
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    valid[e] = base + e * NT < nv;
    key[e] = valid[e] ? float_key(v[e]) : 0u;
  }
  int* out = n_chunks == 1 ? idx_out + (size_t)row * k : cand + ((size_t)row * n_chunks + c) * k;
  const int cnt = block_topk<NT, PT>(key, valid, k, [&](int e) { return base + e * NT; }, out, sh);
  if (n_chunks == 1) {
    for (int i = cnt + threadIdx.x; i < k; i += NT) out[i] = -1;
  } else if (threadIdx.x == 0) {
    cand_n[(size_t)row * n_chunks + c] = cnt;
  }
}

// One CTA per query row: the top-k of the concatenated chunk candidates.
template <int NT, int PT>
__global__ void __launch_bounds__(NT)
    k_topk_merge(const float* __restrict__ scores, int n_max, int k, int n_chunks,
                 const int* __restrict__ cand, const int* __restrict__ cand_n,
                 int* __restrict__ idx_out) {
  __shared__ TopkShared<NT, PT> sh;
  __shared__ int offs[65];
  sm100::griddep_wait();
  sm100::griddep_launch_dependents();
  const int row = blockIdx.x;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int c = 0; c < n_chunks; ++c) {
      offs[c] = acc;
      acc += cand_n[(size_t)row * n_chunks + c];
    }
    offs[n_chunks] = acc;
  }
  __syncthreads();
  const int total = offs[n_chunks];
  const float* s = scores + (size_t)row * n_max;
  uint32_t key[PT];
  bool valid[PT];
  int idx[PT];
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const int p = e * NT + (int)threadIdx.x;
    valid[e] = p < total;
    idx[e] = -1;
    if (valid[e]) {
      int lo = 0, hi = n_chunks - 1;  // last chunk c with offs[c] <= p
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs[mid] <= p) lo = mid; else hi = mid - 1;
      }
      idx[e] = cand[((size_t)row * n_chunks + lo) * k + (p - offs[lo])];
    }
    key[e] = valid[e] ? float_key(s[idx[e]]) : 0u;
  }
  int* out = idx_out + (size_t)row * k;
  const int cnt = block_topk<NT, PT>(key, valid, k, [&](int e) { return idx[e]; }, out, sh);
  for (int i = cnt + threadIdx.x; i < k; i += NT) out[i] = -1;
}

// ---------------------------------------------------------------------------
// Few long rows: one thread-block cluster of C CTAs per row (C = gridDim.x,
// at most MAXC: up to 8 CTAs of 4,096 entries, or up to 16 of 16,384 for
// rows of up to 262,144 entries), CTA c holding entries [c * NT * PT,
// (c + 1) * NT * PT) striped as above.  The CTAs exchange, through distributed shared
// memory, their valid counts and AND/OR of keys, each radix pass's 256-bin
// histogram and, at the end, their counts of greater and boundary keys; one
// cluster barrier per exchange.  Every CTA then takes the same decisions on
// the same totals and places its kept entries after those of the lower
// ranks, so the row's output is the single-block result.
constexpr int kTopkMaxCluster = 8;       // 4,096-entry CTAs (256 x 16), portable cluster
constexpr int kTopkMaxWideCluster = 16;  // 16,384-entry CTAs (1024 x 16), non-portable size

template <int NT, int PT, int MAXC>
struct TopkClusterShared {
  TopkShared<NT, PT> loc;
  unsigned xh[2][MAXC][256];  // per-pass histograms of every rank (double buffer)
  int xv[3][MAXC][3];         // small per-rank values of the three exchanges
};

// Stores v at the same shared-memory offset as `local` in cluster CTA `rank`.
__device__ __forceinline__ void dsmem_store(const void* local, uint32_t rank, uint32_t v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(ra)
               : "r"(sm100::smem_u32(local)), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}

template <int NT, int PT, int MAXC = kTopkMaxCluster>
__global__ void __launch_bounds__(NT)
    k_topk_cluster(const float* __restrict__ scores, const int* __restrict__ q_pos,
                   const int* __restrict__ n_cmp, int Tq, int n_max, int k, int width,
                   int stride, int* __restrict__ idx_out) {
  static_assert(NT >= 256, "bin scan needs 256 threads");
  static_assert(NT * PT < 65536, "per-CTA counts are packed in 16 bits");
  constexpr int NW = NT / 32;
  __shared__ TopkClusterShared<NT, PT, MAXC> sh;
  sm100::griddep_wait();  // the scores of the predecessor are visible
  sm100::griddep_launch_dependents();
  const int C = (int)gridDim.x;
  const int c = (int)blockIdx.x;  // cluster rank: the cluster spans the grid's x
  const int row = blockIdx.y;
  const int b = row / Tq;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int base = c * NT * PT + (int)threadIdx.x;
  const float* s = scores + (size_t)row * n_max;
  int* out = idx_out + (size_t)row * k;
  float v[PT];
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const int j = base + e * NT;
    v[e] = j < n_max ? s[j] : 0.f;
  }
  const int nv = min(n_visible(q_pos[row], n_cmp[b], width, stride), n_max);
  uint32_t key[PT];
  bool valid[PT];
  int nv_local = 0;
  uint32_t k_and = 0xffffffffu, k_or = 0u;
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    valid[e] = base + e * NT < nv;
    key[e] = valid[e] ? float_key(v[e]) : 0u;
    if (valid[e]) {
      ++nv_local;
      k_and &= key[e];
      k_or |= key[e];
    }
  }
  // ---- exchange 0: valid counts and AND / OR of the keys
  int n_mine;
  block_inclusive_scan(nv_local, sh.loc.scan, &n_mine);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
    k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
  }
  if (lane == 0) {
    sh.loc.red_and[wid] = k_and;
    sh.loc.red_or[wid] = k_or;
  }
  __syncthreads();
  if ((int)threadIdx.x < C) {
    uint32_t a = 0xffffffffu, o = 0u;
    for (int w = 0; w < NW; ++w) {
      a &= sh.loc.red_and[w];
      o |= sh.loc.red_or[w];
    }
    const uint32_t r = threadIdx.x;
    dsmem_store(&sh.xv[0][c][0], r, (uint32_t)n_mine);
    dsmem_store(&sh.xv[0][c][1], r, a);
    dsmem_store(&sh.xv[0][c][2], r, o);
  }
  sm100::cluster_sync_all();
  int n_valid = 0, valid_before = 0;
  k_and = 0xffffffffu;
  k_or = 0u;
  for (int r = 0; r < C; ++r) {
    const int n = sh.xv[0][r][0];
    n_valid += n;
    valid_before += r < c ? n : 0;
    if (n > 0) {
      k_and &= (uint32_t)sh.xv[0][r][1];
      k_or |= (uint32_t)sh.xv[0][r][2];
    }
  }
  if (c == 0)
    for (int i = min(n_valid, k) + (int)threadIdx.x; i < k; i += NT) out[i] = -1;
  if (n_valid <= k) {  // keep every valid entry
    place_selected<NT, PT>(valid, k - valid_before, [&](int e) { return base + e * NT; },
                           out + valid_before, sh.loc);
    return;  // no exchange follows: no CTA writes into another's memory any more
  }
  // ---- radix select on the row's totals
  const uint32_t diff = k_and ^ k_or;
  uint32_t prefix, mask;
  int remaining = k;
  if (diff == 0u) {
    prefix = k_and;
    mask = 0xffffffffu;
  } else {
    int hi = 31 - __clz(diff);
    mask = hi == 31 ? 0u : (0xffffffffu << (hi + 1));
    prefix = k_and & mask;
    int pass = 0;
#pragma unroll 1
    while (hi >= 0) {
      const int lo = max(hi - 7, 0);
      const uint32_t dmask = ((hi - lo == 31) ? 0xffffffffu : ((1u << (hi - lo + 1)) - 1u));
      for (int i = threadIdx.x; i < 256; i += NT) sh.loc.hist[i] = 0u;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < PT; ++e)
        if (valid[e] && (key[e] & mask) == prefix)
          atomicAdd(&sh.loc.hist[(key[e] >> lo) & dmask], 1u);
      __syncthreads();
      unsigned (*xh)[256] = sh.xh[pass & 1];
      if (threadIdx.x < 256) {
        const unsigned h = sh.loc.hist[threadIdx.x];
        for (int r = 0; r < C; ++r) dsmem_store(&xh[c][threadIdx.x], (uint32_t)r, h);
      }
      sm100::cluster_sync_all();
      if (threadIdx.x < 256) {
        const int bin = 255 - (int)threadIdx.x;
        int h = 0;
        for (int r = 0; r < C; ++r) h += (int)xh[r][bin];
        int x = h;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += n;
        }
        if (lane == 31) sh.loc.scan[wid] = x;
        asm volatile("bar.sync 3, 256;" ::: "memory");
        int off = 0;
        for (int w = 0; w < wid; ++w) off += sh.loc.scan[w];
        const int incl = off + x, excl = incl - h;
        if (incl >= remaining && excl < remaining) {
          sh.loc.prefix = prefix | ((uint32_t)bin << lo);
          sh.loc.remaining = remaining - excl;
          sh.loc.bin_count = h;
        }
      }
      __syncthreads();
      prefix = sh.loc.prefix;
      remaining = sh.loc.remaining;
      mask |= dmask << lo;
      hi = lo - 1;
      ++pass;
      if (remaining == sh.loc.bin_count) break;  // the boundary bin is kept whole
    }
  }
  // ---- exchange 2: greater and boundary counts of every rank
  int g_mine = 0, q_mine = 0;
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const uint32_t km = key[e] & mask;
    g_mine += (valid[e] && km > prefix) ? 1 : 0;
    q_mine += (valid[e] && km == prefix) ? 1 : 0;
  }
  int g_tot, q_tot;
  block_inclusive_scan(g_mine, sh.loc.scan, &g_tot);
  block_inclusive_scan(q_mine, sh.loc.scan, &q_tot);
  if ((int)threadIdx.x < C) {
    dsmem_store(&sh.xv[2][c][0], threadIdx.x, (uint32_t)g_tot);
    dsmem_store(&sh.xv[2][c][1], threadIdx.x, (uint32_t)q_tot);
  }
  sm100::cluster_sync_all();
  int g_rank = 0, q_rank0 = 0;  // greater / boundary keys in the lower ranks
  for (int r = 0; r < c; ++r) {
    g_rank += sh.xv[2][r][0];
    q_rank0 += sh.xv[2][r][1];
  }
  // ---- placement, as in block_topk, offset by the lower ranks
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const uint32_t km = key[e] & mask;
    const unsigned mg = __ballot_sync(0xffffffffu, valid[e] && km > prefix);
    const unsigned mq = __ballot_sync(0xffffffffu, valid[e] && km == prefix);
    if (lane == 0) sh.loc.cnt[e * NW + wid] = (__popc(mg) << 16) | __popc(mq);
  }
  scan_groups(sh.loc);
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const uint32_t km = key[e] & mask;
    const bool g = valid[e] && km > prefix, q = valid[e] && km == prefix;
    const unsigned mg = __ballot_sync(0xffffffffu, g);
    const unsigned mq = __ballot_sync(0xffffffffu, q);
    const int before = sh.loc.cnt[e * NW + wid];
    const int g_before = g_rank + (before >> 16), q_before = q_rank0 + (before & 0xffff);
    const int q_rank = q_before + __popc(mq & lt);
    if (g || (q && q_rank < remaining)) {
      const int pos = g_before + __popc(mg & lt) + min(q_rank, remaining);
      if (pos < k) out[pos] = base + e * NT;
    }
  }
}

}  // namespace csa
