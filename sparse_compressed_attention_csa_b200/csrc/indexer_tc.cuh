// Step 2a on tensor cores: lightning-indexer scores for the measured shape
// (64 indexer heads x 128 dims, bf16) - "Compressed Sparse Attention" row:
// "64 heads x 128 dims, ReLU scores weighted per head".
//
//   D[key][q*64 + h] = sum_c k_idx[key][c] * q_idx[q][h][c]     (tcgen05, fp32 in TMEM)
//   s[q][key]        = sum_h w[q][h] * max(0, D[key][q*64 + h])  (epilogue, one thread/key)
//
// Keys are the MMA's M (128 per tile), the block's QPB query tokens x 64
// heads its N, the 128 indexer dims its K.  The key scan is HBM-bound
// (256 B per key in, 4 B per key out for decode), so the kernel is a TMA
// pipeline: warp 0 streams key tiles into a STAGES-deep ring of 128B-swizzled
// shared-memory tiles, one thread of warp 1 issues the MMAs into two TMEM
// accumulators, warps 2-5 read the accumulators back (one TMEM lane = one
// key per thread) and write the scores.  Every product and sum is exact for
// integer-valued inputs with power-of-two weights (partial sums < 2^24).
// Decode runs two CTAs per SM with 2-stage rings (measured faster than one
// CTA with a 6-stage ring: the two interleave each other's epilogue and MMA
// latency).
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kIdxTcKeys = 128;
constexpr int kIdxTcHeads = 64;
constexpr int kIdxTcDim = 128;
constexpr int kIdxTcThreads = 192;
constexpr uint64_t kIdxDrainNs = 100000000ull;  // 100 ms for the wind-down waits

template <int QPB, int STAGES>
struct IdxTcSmem {
  static constexpr int kN = QPB * kIdxTcHeads;            // MMA N
  static constexpr int kQBytes = kN * kIdxTcDim * 2;      // B operand
  static constexpr int kKBytes = kIdxTcKeys * kIdxTcDim * 2;  // A operand per stage
  alignas(1024) uint8_t q[kQBytes];             // [2 k-blocks][kN rows][128 B]
  alignas(1024) uint8_t keys[STAGES][kKBytes];  // [2 k-blocks][128 rows][128 B]
  float w[QPB][kIdxTcHeads];
  uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], q_bar;
  uint32_t tmem_base;
  int abort_flag;
};

template <int QPB>
__host__ __device__ constexpr uint32_t idx_tmem_cols() {
  return 2 * QPB * kIdxTcHeads <= 32 ? 32 : (2 * QPB * kIdxTcHeads <= 64 ? 64 :
         (2 * QPB * kIdxTcHeads <= 128 ? 128 : (2 * QPB * kIdxTcHeads <= 256 ? 256 : 512)));
}

template <int QPB, int STAGES>
__global__ void __launch_bounds__(kIdxTcThreads, 1)
    k_index_scores_tc(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_q, const float* __restrict__ w,
                      const int* __restrict__ q_pos, const int* __restrict__ n_cmp, int Tq,
                      int n_max, int width, int stride, int chunks, unsigned long long wait_ns,
                      float* __restrict__ scores) {
  using namespace sm100;
  using S = IdxTcSmem<QPB, STAGES>;
  constexpr int N = S::kN;
  constexpr uint32_t kCols = idx_tmem_cols<QPB>();
  extern __shared__ uint8_t smem_raw[];
  S& sm = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                ~static_cast<uintptr_t>(1023));
  griddep_wait();  // inputs written by the predecessor are visible
  griddep_launch_dependents();
  const int b = blockIdx.y;
  const int qb = blockIdx.x / chunks, chunk = blockIdx.x % chunks;
  const int t0 = qb * QPB;
  const int nq = min(QPB, Tq - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int nv_q[QPB];
  int nv_max = 0;
#pragma unroll
  for (int q = 0; q < QPB; ++q) {
    nv_q[q] = q < nq ? min(n_visible(q_pos[b * Tq + t0 + q], n_cmp[b], width, stride), n_max) : 0;
    nv_max = max(nv_max, nv_q[q]);
  }
  const int tiles = (nv_max + kIdxTcKeys - 1) / kIdxTcKeys;
  const int tb = (int)((long long)tiles * chunk / chunks);
  const int te = (int)((long long)tiles * (chunk + 1) / chunks);
  const int ntile = te - tb;
  if (ntile <= 0) return;  // uniform: nothing allocated yet

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 128);
    }
    mbar_init(&sm.q_bar, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, kCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < QPB * kIdxTcHeads; i += blockDim.x) {
    const int q = i / kIdxTcHeads, h = i % kIdxTcHeads;
    sm.w[q][h] = q < nq ? w[(size_t)(b * Tq + t0 + q) * kIdxTcHeads + h] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abortp = &sm.abort_flag;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_q);
      const int qrow = (b * Tq + t0) * kIdxTcHeads;
      mbar_arrive_expect_tx(&sm.q_bar, S::kQBytes);
      tma_load_2d(sm.q, &tm_q, &sm.q_bar, 0, qrow);
      tma_load_2d(sm.q + S::kQBytes / 2, &tm_q, &sm.q_bar, 64, qrow);
      int issued = 0;
      for (int i = 0; i < ntile; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(&sm.empty[s], ph ^ 1u, abortp, wait_ns)) break;
        mbar_arrive_expect_tx(&sm.full[s], S::kKBytes);
        const int row = b * n_max + (tb + i) * kIdxTcKeys;
        tma_load_2d(sm.keys[s], &tm_k, &sm.full[s], 0, row);
        tma_load_2d(sm.keys[s] + S::kKBytes / 2, &tm_k, &sm.full[s], 64, row);
        issued = i + 1;
      }
      // drain: every issued copy lands before the CTA may exit
      for (int i = max(0, issued - STAGES); i < issued; ++i)
        mbar_drain(&sm.full[i % STAGES], (uint32_t)(i / STAGES) & 1u, kIdxDrainNs);
      mbar_drain(&sm.q_bar, 0, kIdxDrainNs);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, N);
      int last = -1;
      if (mbar_wait(&sm.q_bar, 0, abortp, wait_ns)) {
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm.q);
        for (int i = 0; i < ntile; ++i) {
          const int s = i % STAGES;
          const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
          const int a = i & 1;
          const uint32_t aph = (uint32_t)(i >> 1) & 1u;
          if (!mbar_wait(&sm.acc_empty[a], aph ^ 1u, abortp, wait_ns)) break;
          if (!mbar_wait(&sm.full[s], ph, abortp, wait_ns)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm.keys[s]);
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = sw128_desc(k_addr + kb * (S::kKBytes / 2) + ks * 32, 16, 1024);
              const uint64_t bd = sw128_desc(q_addr + kb * (S::kQBytes / 2) + ks * 32, 16, 1024);
              mma_ss(tmem + (uint32_t)(a * N), ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&sm.empty[s]);
          tc_commit(&sm.acc_full[a]);
          last = i;
        }
      }
      if (last >= 0) {  // the accumulators are released only after the last MMA lands
        mbar_drain(&sm.acc_full[last & 1], (uint32_t)(last >> 1) & 1u, kIdxDrainNs);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quarter = warp % 4
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    for (int i = 0; i < ntile; ++i) {
      const int a = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      bool ok = mbar_wait(&sm.acc_full[a], aph, abortp, wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float sc[QPB];
#pragma unroll
      for (int q = 0; q < QPB; ++q) {
        float s = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(a * N + q * 64 + half * 32), r);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 32; ++h)
            s = fmaf(sm.w[q][half * 32 + h], fmaxf(__uint_as_float(r[h]), 0.f), s);
        }
        sc[q] = s;
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[a]);
      const int j = (tb + i) * kIdxTcKeys + quarter * 32 + lane;
#pragma unroll
      for (int q = 0; q < QPB; ++q)
        if (j < nv_q[q]) scores[(size_t)(b * Tq + t0 + q) * n_max + j] = sc[q];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}


}  // namespace csa
