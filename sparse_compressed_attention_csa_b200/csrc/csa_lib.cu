// C ABI of the CSA library: argument validation, workspace sizing and kernel
// launches.  Declarations and the contract of every call are in csa.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn_pair.cuh"
#include "attn_simt.cuh"
#include "common.cuh"
#include "compress.cuh"
#include "quantize.cuh"
#include "csa.h"
#include "indexer_simt.cuh"
#include "indexer_tc.cuh"
#include "topk.cuh"
#include "topk_block.cuh"

namespace csa {
namespace {

thread_local char g_detail[512] = "";

// Tracing: every call of the C ABI that validates, plans or launches opens an
// NVTX range named after itself, in the domain "csa", for its host-side
// duration.  With no tool attached an NVTX call is one test of a function
// pointer; under Nsight Systems (or any NVTX injection library) the ranges
// show which call launched which kernels.
nvtxDomainHandle_t trace_domain() {
  static const nvtxDomainHandle_t d = nvtxDomainCreateA("csa");
  return d;
}

struct CallRange {
  explicit CallRange(const char* name) {
    nvtxEventAttributes_t ev;
    std::memset(&ev, 0, sizeof(ev));
    ev.version = NVTX_VERSION;
    ev.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    ev.messageType = NVTX_MESSAGE_TYPE_ASCII;
    ev.message.ascii = name;
    nvtxDomainRangePushEx(trace_domain(), &ev);
  }
  ~CallRange() { nvtxDomainRangePop(trace_domain()); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

csa_status_t fail(csa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return st;
}

csa_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(CSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define CSA_CHECK(expr)                  \
  do {                                   \
    csa_status_t _s = (expr);            \
    if (_s != CSA_OK) return _s;         \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

csa_status_t check_ptr(const void* p, const char* name, bool nullable = false) {
  if (p == nullptr) {
    if (nullable) return CSA_OK;
    return fail(CSA_ERR_INVALID_ARGUMENT, "%s is NULL", name);
  }
  if (!aligned16(p)) return fail(CSA_ERR_MISALIGNED, "%s is not 16-byte aligned", name);
  return CSA_OK;
}

csa_status_t check_device() {
  static int checked[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= 0 && dev < 64 && checked[dev] == 1) return CSA_OK;
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10) {
    if (dev >= 0 && dev < 64) checked[dev] = 2;
    return fail(CSA_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d0, the library is built for sm_100a",
                dev, major);
  }
  if (dev >= 0 && dev < 64) checked[dev] = 1;
  return CSA_OK;
}

csa_status_t check_params(const csa_params_t* p) {
  if (p == nullptr) return fail(CSA_ERR_INVALID_ARGUMENT, "params is NULL");
  if (p->d != 64 && p->d != 128 && p->d != 256 && p->d != 512 && p->d != 1024)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "d=%d: supported 64, 128, 256, 512, 1024", p->d);
  if (p->rope_dim < 0 || p->rope_dim > p->d || (p->rope_dim & 1) || ((p->d - p->rope_dim) & 31))
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "rope_dim=%d: must be even, <= d and leave a multiple of 32 unrotated dims",
                p->rope_dim);
  if (!(p->theta > 0.f) || !std::isfinite(p->theta))
    return fail(CSA_ERR_INVALID_ARGUMENT, "theta must be positive and finite");
  if (!std::isfinite(p->scale)) return fail(CSA_ERR_INVALID_ARGUMENT, "scale must be finite");
  if (p->n_heads < 1 || p->n_heads > 65535)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "n_heads=%d out of [1, 65535]", p->n_heads);
  if (p->width < 1 || p->stride < 1)
    return fail(CSA_ERR_INVALID_ARGUMENT, "width=%d stride=%d must be >= 1", p->width, p->stride);
  if (p->window < 0) return fail(CSA_ERR_INVALID_ARGUMENT, "window=%d < 0", p->window);
  if (!std::isfinite(p->rope_factor))
    return fail(CSA_ERR_INVALID_ARGUMENT, "rope_factor must be finite");
  if (p->rope_factor > 1.f &&
      (p->rope_orig_ctx < 1 || !std::isfinite(p->rope_beta_fast) ||
       !std::isfinite(p->rope_beta_slow) || !(p->rope_beta_fast > p->rope_beta_slow)))
    return fail(CSA_ERR_INVALID_ARGUMENT,
                "YaRN (rope_factor %g > 1) needs rope_orig_ctx >= 1 and rope_beta_fast > "
                "rope_beta_slow (got %d, %g, %g)",
                (double)p->rope_factor, p->rope_orig_ctx, (double)p->rope_beta_fast,
                (double)p->rope_beta_slow);
  return CSA_OK;
}

// The call's RoPE: plain, or YaRN when rope_factor > 1.
RopeSpec rope_spec(const csa_params_t* p) {
  RopeSpec r;
  r.rope_dim = p->rope_dim;
  r.theta = (double)p->theta;
  r.factor = p->rope_factor > 1.f ? (double)p->rope_factor : 1.0;
  r.orig_ctx = (double)p->rope_orig_ctx;
  r.beta_fast = (double)p->rope_beta_fast;
  r.beta_slow = (double)p->rope_beta_slow;
  return r;
}

// Softmax scale of the attention calls: `scale`, times YaRN's temperature
// (0.1 ln s + 1)^2 under the extended RoPE.
float attn_scale(const csa_params_t* p) {
  if (!(p->rope_factor > 1.f)) return p->scale;
  const double m = 0.1 * std::log((double)p->rope_factor) + 1.0;
  return (float)((double)p->scale * m * m);
}

csa_status_t check_indexer_shape(const csa_params_t* p) {
  if (p->idx_heads < 1 || p->idx_dim < 2 || (p->idx_dim & 1) ||
      p->idx_heads * p->idx_dim > 16384)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "idx_heads=%d idx_dim=%d: need idx_dim even and idx_heads*idx_dim <= 16384",
                p->idx_heads, p->idx_dim);
  return CSA_OK;
}

csa_status_t check_topk(const csa_params_t* p) {
  if (p->topk < 1 || p->topk > (1 << 20))
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "topk=%d out of [1, 2^20]", p->topk);
  return CSA_OK;
}

csa_status_t check_dtype(csa_dtype_t dt) {
  if (dt != CSA_F32 && dt != CSA_BF16) return fail(CSA_ERR_INVALID_ARGUMENT, "bad dtype %d", dt);
  return CSA_OK;
}

csa_status_t check_sizes(int B, int Tq, int n_max) {
  // query rows (B * Tq) index a grid dimension of at most 65535 blocks
  if (B < 1 || Tq < 1 || n_max < 0 || (long long)B * Tq > 65535)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "B=%d Tq=%d n_max=%d out of range (B*Tq <= 65535)",
                B, Tq, n_max);
  return CSA_OK;
}

std::atomic<unsigned long long> g_launches{0};

csa_status_t launched(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return CSA_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launch with programmatic dependent launch allowed (the kernel may start
// while its predecessor in the stream finishes; it waits for it in
// griddep_wait() before touching global memory) and, when cluster_x > 1,
// as clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int num_sms() {
  static int cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// Opt a kernel into `bytes` of dynamic shared memory, once per (kernel,
// device).
template <typename K>
csa_status_t set_smem_attr(K* kernel, size_t bytes, const char* name) {
  struct Entry {
    const void* fn;
    int dev;
  };
  static Entry done[256];
  static int n_done = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].fn == (const void*)kernel && done[i].dev == dev) return CSA_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return cuda_fail(e, name);
  // these kernels live on shared memory: ask for the largest carveout, so
  // that occupancy queries and launches both see every CTA that fits
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return cuda_fail(e, name);
  if (n_done < 256) done[n_done++] = Entry{(const void*)kernel, dev};
  return CSA_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// libcuda link dependency).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 tensor map over [rows][inner] row-major, box [box_rows][box_inner],
// 128-byte swizzle (box_inner * 2 must be 128).
csa_status_t make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                            uint32_t box_inner, uint32_t box_rows,
                            CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return fail(CSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CSA_OK;
}

// Row-gather map over E4M3 codes [rows][inner] (bytes), no swizzle.
csa_status_t make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                          uint32_t box_inner) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return fail(CSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CSA_OK;
}

size_t scores_bytes(int B, int Tq, int n_max) {
  return round_up((size_t)B * Tq * (size_t)n_max * sizeof(float), 256);
}

// Top-k plan.  A block holds its candidates in registers: 2048 (256 x 8),
// 4096 (256 x 16) or 16384 (1024 x 16) entries.  Few rows of up to 32768
// entries: one cluster of 4096-entry CTAs per row.  Else one block per row
// when the row fits; two
// stages (per-chunk top-k into a candidate list, then one merge block per
// row over the concatenated candidates) for longer rows when the merge fits
// one block (4096, 8192 or 16384 candidates); else the generic
// shared-memory radix select.  (Splitting rows that fit one block over more
// chunks, to occupy more SMs when rows are few, measured slower: a block's
// select costs about the same for 4096 entries as for 16384.)
struct TopkPlan {
  int chunks;     // 0: generic; 1: single stage; >1: chunk + merge
  int chunk_len;  // entries per chunk block
  int merge_cap;  // candidates per merge block
  int cluster;    // > 1: one cluster of this many CTAs per row, of chunk_len entries each
};

// Whether a cluster of `c` 1024-thread top-k CTAs (a non-portable size
// above 8) can be resident on this device; asked once per device and size.
static bool wide_topk_cluster_fits(int c) {
  static signed char known[64][kTopkMaxWideCluster + 1];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || c < 2 || c > kTopkMaxWideCluster) return false;
  if (known[dev][c]) return known[dev][c] > 0;
  auto kern = k_topk_cluster<1024, 16, kTopkMaxWideCluster>;
  bool ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)c, 1);
    cfg.blockDim = dim3(1024);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)c;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0;
  }
  cudaGetLastError();  // a refusal above is an answer, not an error to keep
  known[dev][c] = ok ? 1 : -1;
  return ok;
}
constexpr int kTopkSmall = 256 * 8, kTopkMid = 256 * 16, kTopkBig = 1024 * 16;

TopkPlan topk_plan(const csa_params_t* p, int B, int Tq, int n_max) {
  const long long rows = (long long)B * Tq;
  const long long k = p->topk;
  // few long rows: a cluster of CTAs per row, so that the SMs share the rows
  if (n_max > kTopkMid && n_max <= kTopkMaxCluster * kTopkMid && 2 * rows <= num_sms()) {
    const int c = (n_max + kTopkMid - 1) / kTopkMid;
    if (rows * c <= num_sms()) return {1, kTopkMid, 0, c};
  }
  // few long rows (or too many rows for clusters of 4,096-entry CTAs): a
  // cluster of up to 16 CTAs of 16,384 entries per row
  if (n_max > kTopkBig && n_max <= kTopkMaxWideCluster * kTopkBig) {
    const int c = (n_max + kTopkBig - 1) / kTopkBig;
    if (rows * c <= num_sms() && wide_topk_cluster_fits(c)) return {1, kTopkBig, 0, c};
  }
  if (n_max <= kTopkSmall) return {1, kTopkSmall, 0, 0};
  if (n_max <= kTopkBig) return {1, kTopkBig, 0, 0};
  const long long c = (n_max + kTopkBig - 1) / kTopkBig;
  if (c <= 64 && c * k <= kTopkBig) {
    const long long cand = c * k;
    return {(int)c, kTopkBig,
            cand <= kTopkMid ? kTopkMid : (cand <= 2 * kTopkMid ? 2 * kTopkMid : kTopkBig), 0};
  }
  return {0, 0, 0, 0};
}

size_t topk_ws_bytes(const csa_params_t* p, int B, int Tq, int n_max) {
  const int c = topk_plan(p, B, Tq, n_max).chunks;
  if (c <= 1) return 0;
  const size_t rows = (size_t)B * Tq;
  return round_up(rows * c * (size_t)p->topk * sizeof(int), 256) +
         round_up(rows * c * sizeof(int), 256);
}


// Tensor-core attention applies to the measured head shape in bf16.
bool attn_tc_ok(const csa_params_t* p, csa_dtype_t dtype, bool hca, int n_max) {
  if (dtype != CSA_BF16 || p->d != kApDim || p->n_heads != kApHeads) return false;
  if (p->rope_dim > kApMaxRope) return false;
  const long long rows = (long long)(hca ? n_max : p->topk) + p->window;
  return rows + 8 <= kApRowCap;
}

// KV splits per query token: each token is a pair of CTAs (one cluster),
// and its splits are further pairs, merged by k_attn_merge.  Enough pairs to
// cover the SMs once, at least two 64-row tiles per split (a split's fixed
// costs - q, the row list, writing 128 KB of partial O - want rows to
// spread over), at most kApMaxSplits.
int attn_splits(const csa_params_t* p, bool hca, int B, int Tq, int n_max) {
  const long long pairs = (long long)B * Tq;
  const long long rows = (long long)(hca ? n_max : p->topk) + p->window;
  long long s = num_sms() / (2 * pairs);
  const long long max_s = (rows + 2 * kApTile - 1) / (2 * kApTile);
  if (s > max_s) s = max_s;
  if (s > kApMaxSplits) s = kApMaxSplits;
  return s < 1 ? 1 : (int)s;
}

size_t attn_ws_bytes(const csa_params_t* p, csa_dtype_t dtype, bool hca, int B, int Tq,
                     int n_max) {
  if (!attn_tc_ok(p, dtype, hca, n_max)) return 0;
  const int sp = attn_splits(p, hca, B, Tq, n_max);
  if (sp == 1) return 0;
  const size_t units = (size_t)B * Tq * sp * 2;  // (token, split, part)
  return round_up(units * kApHeads * kApHalf * sizeof(__half), 256) +
         round_up(units * 2 * kApHeads * sizeof(float), 256);
}

// Limit of every bounded device-side wait (csa_set_wait_limit_ns).
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};

}  // namespace
}  // namespace csa

using namespace csa;

#define CSA_API extern "C" __attribute__((visibility("default")))

CSA_API int csa_abi_version(void) { return CSA_ABI_VERSION; }

CSA_API const char* csa_status_string(csa_status_t s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARGUMENT: return "CSA_ERR_INVALID_ARGUMENT";
    case CSA_ERR_MISALIGNED: return "CSA_ERR_MISALIGNED";
    case CSA_ERR_UNSUPPORTED_SHAPE: return "CSA_ERR_UNSUPPORTED_SHAPE";
    case CSA_ERR_UNSUPPORTED_DEVICE: return "CSA_ERR_UNSUPPORTED_DEVICE";
    case CSA_ERR_WORKSPACE_TOO_SMALL: return "CSA_ERR_WORKSPACE_TOO_SMALL";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_DEVICE_TIMEOUT: return "CSA_ERR_DEVICE_TIMEOUT";
    case CSA_ERR_DEVICE_BOUNDS: return "CSA_ERR_DEVICE_BOUNDS";
  }
  return "CSA_ERR_UNKNOWN";
}

CSA_API const char* csa_last_error_detail(void) { return g_detail; }

CSA_API void csa_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns == 0 ? kDefaultWaitNs : (unsigned long long)ns, std::memory_order_relaxed);
}

CSA_API uint64_t csa_launch_count(void) {
  return g_launches.load(std::memory_order_relaxed);
}

CSA_API csa_status_t csa_workspace_size(const csa_params_t* p, csa_op_t op, int32_t B, int32_t Tq,
                                int32_t n_max, size_t* bytes) {
  const CallRange trace("csa_workspace_size");
  if (bytes == nullptr) return fail(CSA_ERR_INVALID_ARGUMENT, "bytes is NULL");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_sizes(B, Tq, n_max));
  switch (op) {
    case CSA_OP_COMPRESS: *bytes = 0; return CSA_OK;
    case CSA_OP_TOPK_SELECT: *bytes = topk_ws_bytes(p, B, Tq, n_max); return CSA_OK;
    case CSA_OP_INDEX_TOPK:
      *bytes = scores_bytes(B, Tq, n_max) + topk_ws_bytes(p, B, Tq, n_max);
      return CSA_OK;
    case CSA_OP_SPARSE_ATTN: *bytes = attn_ws_bytes(p, CSA_BF16, false, B, Tq, n_max); return CSA_OK;
    case CSA_OP_HCA_ATTN: *bytes = attn_ws_bytes(p, CSA_BF16, true, B, Tq, n_max); return CSA_OK;
  }
  return fail(CSA_ERR_INVALID_ARGUMENT, "bad op %d", (int)op);
}

// e_slots: entries per sequence the launch covers; a.n_raw: raw rows.
static csa_status_t launch_compress(CompressArgs& a, int e_slots, csa_dtype_t dtype, int B,
                                    cudaStream_t s) {
  if (a.rope.rope_dim / 2 > kCompressMaxPairs)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "rope_dim=%d", a.rope.rope_dim);
  for (int i = 0; i < kCompressMaxPairs; ++i)
    a.freq[i] = i < a.rope.rope_dim / 2 ? rope_freq(a.rope, i) : 0.0;
  const bool wide = a.width >= kCompressWideMin;
  a.wide_ctas = wide ? e_slots : 0;
  a.narrow_slots = wide ? 0 : e_slots;
  a.raw_slots = (a.n_raw + kCompressRawPer - 1) / kCompressRawPer;
  const int vec = dtype == CSA_BF16 ? 8 : 4;
  const int rpc = kCompressThreads / (a.d / vec);
  const long long ctas =
      a.wide_ctas + ((long long)a.narrow_slots + a.raw_slots + rpc - 1) / rpc;
  if (ctas == 0) return CSA_OK;
  if (ctas > 2147483647LL) return fail(CSA_ERR_UNSUPPORTED_SHAPE, "too many rows");
  dim3 grid((unsigned)ctas, (unsigned)B);
  if (dtype == CSA_BF16)
    k_compress<__nv_bfloat16><<<grid, kCompressThreads, 0, s>>>(a);
  else
    k_compress<float><<<grid, kCompressThreads, 0, s>>>(a);
  return launched("k_compress");
}

static CompressArgs compress_args(const csa_params_t* p, const void* x, const void* gate) {
  CompressArgs a{};
  a.x = x;
  a.g = gate;
  a.d = p->d;
  a.width = p->width;
  a.stride = p->stride;
  a.pos_offset = p->pos_offset;
  a.rope = rope_spec(p);
  return a;
}

CSA_API csa_status_t csa_compress(const csa_params_t* p, csa_dtype_t dtype, const void* x,
                          const void* gate, int32_t B, int32_t T, void* kv_cmp_out,
                          void* kv_raw_rot_out, void* stream) {
  const CallRange trace("csa_compress");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_dtype(dtype));
  CSA_CHECK(check_ptr(x, "x"));
  CSA_CHECK(check_ptr(gate, "gate"));
  CSA_CHECK(check_ptr(kv_raw_rot_out, "kv_raw_rot_out", true));
  if (B < 1 || B > 65535 || T < 0) return fail(CSA_ERR_UNSUPPORTED_SHAPE, "B=%d T=%d", B, T);
  const int N = T < p->width ? 0 : (T - p->width) / p->stride + 1;
  if (N > 0) CSA_CHECK(check_ptr(kv_cmp_out, "kv_cmp_out"));
  CSA_CHECK(check_device());
  CompressArgs a = compress_args(p, x, gate);
  a.L = T;
  a.T = T;
  a.max_new = T;
  a.n_raw = kv_raw_rot_out ? T : 0;
  a.kv_cmp = kv_cmp_out;
  a.n_cap = N;
  a.kv_raw = kv_raw_rot_out;
  a.raw_cap = T;
  return launch_compress(a, N, dtype, B, (cudaStream_t)stream);
}

CSA_API csa_status_t csa_compress_append(const csa_params_t* p, csa_dtype_t dtype, const void* x,
                                         const void* gate, const int32_t* x_pos0, int32_t B,
                                         int32_t L, const int32_t* t_old, const int32_t* t_new,
                                         int32_t max_new, void* kv_cmp, int32_t n_cap,
                                         void* kv_raw, const int32_t* raw_pos0, int32_t raw_cap,
                                         void* stream) {
  const CallRange trace("csa_compress_append");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_dtype(dtype));
  if (B < 1 || B > 65535 || L < 0 || max_new < 0 || n_cap < 0 || raw_cap < 0)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "B=%d L=%d max_new=%d n_cap=%d raw_cap=%d", B, L,
                max_new, n_cap, raw_cap);
  CSA_CHECK(check_ptr(x, "x", L == 0));
  CSA_CHECK(check_ptr(gate, "gate", L == 0));
  CSA_CHECK(check_ptr(x_pos0, "x_pos0"));
  CSA_CHECK(check_ptr(t_old, "t_old"));
  CSA_CHECK(check_ptr(t_new, "t_new"));
  CSA_CHECK(check_ptr(kv_cmp, "kv_cmp", n_cap == 0));
  CSA_CHECK(check_ptr(kv_raw, "kv_raw", true));
  if (kv_raw) CSA_CHECK(check_ptr(raw_pos0, "raw_pos0"));
  CSA_CHECK(check_device());
  CompressArgs a = compress_args(p, x, gate);
  a.x_pos0 = x_pos0;
  a.L = L;
  a.t_old = t_old;
  a.t_new = t_new;
  a.max_new = max_new;
  // entries completed by max_new consecutive tokens: at most ceil(max_new / stride)
  int e_slots = (int)(((long long)max_new + p->stride - 1) / p->stride);
  a.n_raw = kv_raw ? max_new : 0;
  if (e_slots + a.n_raw == 0) e_slots = 1;  // one CTA still checks t_new - t_old
  a.kv_cmp = kv_cmp;
  a.n_cap = n_cap;
  a.kv_raw = kv_raw;
  a.raw_pos0 = raw_pos0;
  a.raw_cap = raw_cap;
  return launch_compress(a, e_slots, dtype, B, (cudaStream_t)stream);
}

template <int QPB, int STAGES>
static csa_status_t launch_index_tc(const void* q_idx, const float* w, const void* k_idx,
                                    const int32_t* q_pos, const int32_t* n_cmp, int32_t B,
                                    int32_t Tq, int32_t n_max, int width, int stride,
                                    float* scores, cudaStream_t s) {
  CUtensorMap tk, tq;
  CSA_CHECK(make_tmap_bf16(&tk, k_idx, kIdxTcDim, (uint64_t)B * n_max, 64, kIdxTcKeys));
  CSA_CHECK(make_tmap_bf16(&tq, q_idx, kIdxTcDim, (uint64_t)B * Tq * kIdxTcHeads, 64,
                           QPB * kIdxTcHeads));
  const size_t smem = sizeof(IdxTcSmem<QPB, STAGES>) + 1024;
  CSA_CHECK(set_smem_attr(k_index_scores_tc<QPB, STAGES>, smem, "k_index_scores_tc"));
  const int qblocks = (Tq + QPB - 1) / QPB;
  // key ranges per query block: enough CTAs to fill every SM with as many
  // CTAs as its 228 KB of shared memory holds (1 KB reserved per CTA); the
  // registers (192 threads x at most 168) allow two
  const int per_sm = 2 * (smem + 1024) <= 228 * 1024 ? 2 : 1;
  const int slots = per_sm * num_sms();
  int chunks = 1;
  if (qblocks * B < slots) chunks = slots / (qblocks * B);
  dim3 grid((unsigned)(qblocks * chunks), (unsigned)B);
  const cudaError_t e = launch_ex(k_index_scores_tc<QPB, STAGES>, grid, dim3(kIdxTcThreads), smem,
                                  s, 1, tk, tq, w, q_pos, n_cmp, Tq, n_max, width, stride, chunks,
                                  g_wait_ns.load(std::memory_order_relaxed), scores);
  if (e != cudaSuccess) return cuda_fail(e, "k_index_scores_tc");
  return launched("k_index_scores_tc");
}

static csa_status_t index_scores_impl(const csa_params_t* p, csa_dtype_t dtype, const void* q_idx,
                                      const float* w, const void* k_idx, const int32_t* q_pos,
                                      const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                                      float* scores, cudaStream_t s) {
  if (n_max == 0) return CSA_OK;
  const int H_I = p->idx_heads, d_I = p->idx_dim;
  // tensor-core path: the measured indexer shape in bf16
  if (dtype == CSA_BF16 && H_I == kIdxTcHeads && d_I == kIdxTcDim &&
      (long long)B * n_max >= kIdxTcKeys) {
    if (Tq == 1)
      return launch_index_tc<1, 2>(q_idx, w, k_idx, q_pos, n_cmp, B, Tq, n_max, p->width,
                                   p->stride, scores, s);
    if ((long long)B * Tq >= 2)
      return launch_index_tc<2, 2>(q_idx, w, k_idx, q_pos, n_cmp, B, Tq, n_max, p->width,
                                   p->stride, scores, s);
  }
  dim3 grid((unsigned)((n_max + kIdxSimtKeys - 1) / kIdxSimtKeys), (unsigned)Tq, (unsigned)B);
  const size_t smem = (size_t)(H_I * d_I + H_I) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e;
    if (dtype == CSA_BF16)
      e = cudaFuncSetAttribute(k_index_scores_simt<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else
      e = cudaFuncSetAttribute(k_index_scores_simt<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(k_index_scores_simt)");
  }
  if (dtype == CSA_BF16)
    k_index_scores_simt<__nv_bfloat16><<<grid, kIdxSimtKeys, smem, s>>>(
        (const __nv_bfloat16*)q_idx, w, (const __nv_bfloat16*)k_idx, q_pos, n_cmp, Tq, n_max,
        H_I, d_I, p->width, p->stride, scores);
  else
    k_index_scores_simt<float><<<grid, kIdxSimtKeys, smem, s>>>(
        (const float*)q_idx, w, (const float*)k_idx, q_pos, n_cmp, Tq, n_max, H_I, d_I,
        p->width, p->stride, scores);
  return launched("k_index_scores_simt");
}

static csa_status_t topk_impl(const csa_params_t* p, const float* scores, const int32_t* q_pos,
                              const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                              int32_t* idx_out, void* ws, size_t ws_bytes, cudaStream_t s) {
  const unsigned rows = (unsigned)B * (unsigned)Tq;
  const int k = p->topk;
  const TopkPlan plan = topk_plan(p, B, Tq, n_max);
  const int chunks = plan.chunks;
  int* none = nullptr;
  if (plan.cluster > 1) {
    const cudaError_t e =
        plan.chunk_len == kTopkMid
            ? launch_ex(k_topk_cluster<256, 16>, dim3((unsigned)plan.cluster, rows), dim3(256), 0,
                        s, plan.cluster, scores, q_pos, n_cmp, Tq, n_max, k, p->width, p->stride,
                        idx_out)
            : launch_ex(k_topk_cluster<1024, 16, kTopkMaxWideCluster>,
                        dim3((unsigned)plan.cluster, rows), dim3(1024), 0, s, plan.cluster, scores,
                        q_pos, n_cmp, Tq, n_max, k, p->width, p->stride, idx_out);
    if (e != cudaSuccess) return cuda_fail(e, "k_topk_cluster");
    return launched("k_topk_cluster");
  }
  if (chunks == 1) {
    const cudaError_t e =
        plan.chunk_len == kTopkSmall
            ? launch_ex(k_topk_chunk<256, 8>, dim3(1, rows), dim3(256), 0, s, 1, scores, q_pos,
                        n_cmp, Tq, n_max, k, p->width, p->stride, 1, idx_out, none, none)
            : launch_ex(k_topk_chunk<1024, 16>, dim3(1, rows), dim3(1024), 0, s, 1, scores, q_pos,
                        n_cmp, Tq, n_max, k, p->width, p->stride, 1, idx_out, none, none);
    if (e != cudaSuccess) return cuda_fail(e, "k_topk_chunk");
    return launched("k_topk_chunk");
  }
  if (chunks > 1) {
    const size_t need = topk_ws_bytes(p, B, Tq, n_max);
    if (ws_bytes < need)
      return fail(CSA_ERR_WORKSPACE_TOO_SMALL, "top-k workspace %zu bytes, need %zu", ws_bytes,
                  need);
    CSA_CHECK(check_ptr(ws, "ws"));
    int* cand = (int*)ws;
    int* cand_n = (int*)((char*)ws + round_up((size_t)rows * chunks * (size_t)k * sizeof(int), 256));
    cudaError_t e = launch_ex(k_topk_chunk<1024, 16>, dim3((unsigned)chunks, rows), dim3(1024), 0,
                              s, 1, scores, q_pos, n_cmp, Tq, n_max, k, p->width, p->stride,
                              chunks, idx_out, cand, cand_n);
    if (e != cudaSuccess) return cuda_fail(e, "k_topk_chunk");
    CSA_CHECK(launched("k_topk_chunk"));
    if (plan.merge_cap == kTopkMid)
      e = launch_ex(k_topk_merge<256, 16>, dim3(rows), dim3(256), 0, s, 1, scores, n_max, k,
                    chunks, cand, cand_n, idx_out);
    else if (plan.merge_cap == 2 * kTopkMid)
      e = launch_ex(k_topk_merge<512, 16>, dim3(rows), dim3(512), 0, s, 1, scores, n_max, k,
                    chunks, cand, cand_n, idx_out);
    else
      e = launch_ex(k_topk_merge<1024, 16>, dim3(rows), dim3(1024), 0, s, 1, scores, n_max, k,
                    chunks, cand, cand_n, idx_out);
    if (e != cudaSuccess) return cuda_fail(e, "k_topk_merge");
    return launched("k_topk_merge");
  }
  k_topk_rows<1024><<<rows, 1024, 0, s>>>(scores, q_pos, n_cmp, Tq, n_max, k, p->width,
                                          p->stride, idx_out);
  return launched("k_topk_rows");
}

CSA_API csa_status_t csa_index_scores(const csa_params_t* p, csa_dtype_t dtype, const void* q_idx,
                              const float* w, const void* k_idx, const int32_t* q_pos,
                              const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                              float* scores, void* stream) {
  const CallRange trace("csa_index_scores");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_dtype(dtype));
  CSA_CHECK(check_indexer_shape(p));
  CSA_CHECK(check_sizes(B, Tq, n_max));
  CSA_CHECK(check_ptr(q_idx, "q_idx"));
  CSA_CHECK(check_ptr(w, "w"));
  CSA_CHECK(check_ptr(k_idx, "k_idx", n_max == 0));
  CSA_CHECK(check_ptr(q_pos, "q_pos"));
  CSA_CHECK(check_ptr(n_cmp, "n_cmp"));
  CSA_CHECK(check_ptr(scores, "scores", n_max == 0));
  CSA_CHECK(check_device());
  return index_scores_impl(p, dtype, q_idx, w, k_idx, q_pos, n_cmp, B, Tq, n_max, scores,
                           (cudaStream_t)stream);
}

CSA_API csa_status_t csa_topk_select(const csa_params_t* p, const float* scores, const int32_t* q_pos,
                             const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                             int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  const CallRange trace("csa_topk_select");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_topk(p));
  CSA_CHECK(check_sizes(B, Tq, n_max));
  CSA_CHECK(check_ptr(scores, "scores", n_max == 0));
  CSA_CHECK(check_ptr(q_pos, "q_pos"));
  CSA_CHECK(check_ptr(n_cmp, "n_cmp"));
  CSA_CHECK(check_ptr(idx_out, "idx_out"));
  CSA_CHECK(check_ptr(ws, "ws", true));
  CSA_CHECK(check_device());
  return topk_impl(p, scores, q_pos, n_cmp, B, Tq, n_max, idx_out, ws, ws_bytes,
                   (cudaStream_t)stream);
}

CSA_API csa_status_t csa_index_topk(const csa_params_t* p, csa_dtype_t dtype, const void* q_idx,
                            const float* w, const void* k_idx, const int32_t* q_pos,
                            const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                            int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  const CallRange trace("csa_index_topk");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_dtype(dtype));
  CSA_CHECK(check_indexer_shape(p));
  CSA_CHECK(check_topk(p));
  CSA_CHECK(check_sizes(B, Tq, n_max));
  CSA_CHECK(check_ptr(q_idx, "q_idx"));
  CSA_CHECK(check_ptr(w, "w"));
  CSA_CHECK(check_ptr(k_idx, "k_idx", n_max == 0));
  CSA_CHECK(check_ptr(q_pos, "q_pos"));
  CSA_CHECK(check_ptr(n_cmp, "n_cmp"));
  CSA_CHECK(check_ptr(idx_out, "idx_out"));
  const size_t sb = scores_bytes(B, Tq, n_max);
  const size_t need = sb + topk_ws_bytes(p, B, Tq, n_max);
  if (need > 0) CSA_CHECK(check_ptr(ws, "ws"));
  if (ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes, need %zu", ws_bytes, need);
  CSA_CHECK(check_device());
  cudaStream_t s = (cudaStream_t)stream;
  float* scores = (float*)ws;
  CSA_CHECK(index_scores_impl(p, dtype, q_idx, w, k_idx, q_pos, n_cmp, B, Tq, n_max, scores, s));
  return topk_impl(p, scores, q_pos, n_cmp, B, Tq, n_max, idx_out, (char*)ws + sb, ws_bytes - sb,
                   s);
}

static csa_status_t attn_common_checks(const csa_params_t* p, csa_dtype_t dtype, const void* q,
                                       const int32_t* q_pos, const void* kv_cmp, int32_t n_max,
                                       const void* kv_raw, const int32_t* raw_pos0,
                                       const int32_t* n_raw, int32_t raw_max, const float* sink,
                                       int32_t B, int32_t Tq, void* out) {
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_dtype(dtype));
  CSA_CHECK(check_sizes(B, Tq, n_max));
  if (raw_max < 0) return fail(CSA_ERR_INVALID_ARGUMENT, "raw_max=%d < 0", raw_max);
  CSA_CHECK(check_ptr(q, "q"));
  CSA_CHECK(check_ptr(q_pos, "q_pos"));
  CSA_CHECK(check_ptr(kv_cmp, "kv_cmp", n_max == 0));
  CSA_CHECK(check_ptr(kv_raw, "kv_raw", raw_max == 0));
  CSA_CHECK(check_ptr(raw_pos0, "raw_pos0"));
  CSA_CHECK(check_ptr(n_raw, "n_raw"));
  CSA_CHECK(check_ptr(sink, "sink"));
  return check_ptr(out, "out");
}

template <bool kHca>
static csa_status_t launch_attn_simt(const AttnArgs& a, csa_dtype_t dtype, cudaStream_t s) {
  dim3 grid((unsigned)a.H, (unsigned)a.Tq, (unsigned)a.B);
  const int nk = a.d / 32;
#define CSA_ATTN_CASE(NKV)                                                        \
  case NKV:                                                                       \
    if (dtype == CSA_BF16)                                                        \
      k_attn_simt<__nv_bfloat16, kHca, NKV><<<grid, 32 * kAttnSimtWarps, 0, s>>>(a); \
    else                                                                          \
      k_attn_simt<float, kHca, NKV><<<grid, 32 * kAttnSimtWarps, 0, s>>>(a);      \
    break;
  switch (nk) {
    CSA_ATTN_CASE(2)
    CSA_ATTN_CASE(4)
    CSA_ATTN_CASE(8)
    CSA_ATTN_CASE(16)
    CSA_ATTN_CASE(32)
    default: return fail(CSA_ERR_UNSUPPORTED_SHAPE, "d=%d", a.d);
  }
#undef CSA_ATTN_CASE
  return launched("k_attn_simt");
}

template <bool kHca, bool kFp8 = false>
static csa_status_t launch_attn_tc(const csa_params_t* p, const AttnArgs& g, void* ws,
                                   size_t ws_bytes, cudaStream_t s) {
  const int LB = g.layers * g.B;  // (layer, sequence) rows of the grid
  const int sp = attn_splits(p, kHca, LB, g.Tq, g.n_max);
  const size_t need = attn_ws_bytes(p, CSA_BF16, kHca, LB, g.Tq, g.n_max);
  if (ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes, need %zu", ws_bytes, need);
  if (need > 0) CSA_CHECK(check_ptr(ws, "ws"));
  AttnPairArgs a;
  a.q = (const __nv_bfloat16*)g.q;
  a.q_pos = g.q_pos;
  a.kv_cmp = (const __nv_bfloat16*)g.kv_cmp;
  a.idx = g.idx;
  a.n_cmp = g.n_cmp;
  a.n_max = g.n_max;
  a.kv_raw = (const __nv_bfloat16*)g.kv_raw;
  a.cmp_scale = g.cmp_scale;
  a.raw_scale = g.raw_scale;
  a.raw_pos0 = g.raw_pos0;
  a.n_raw = g.n_raw;
  a.raw_max = g.raw_max;
  a.sink = g.sink;
  a.Tq = g.Tq;
  a.rows_per_layer = g.B * g.Tq;
  a.topk = g.topk;
  a.window = g.window;
  a.width = g.width;
  a.stride = g.stride;
  a.rope_dim = g.rope_dim;
  a.scale_log2 = g.scale * 1.4426950408889634f;
  a.splits = sp;
  a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  a.out = (__nv_bfloat16*)g.out;
  a.part_o = nullptr;
  a.part_ml = nullptr;
  if (sp > 1) {
    // workspace: partial O | partial (m, l)
    const size_t units = (size_t)LB * g.Tq * sp * 2;
    const size_t o_bytes = round_up(units * kApHeads * kApHalf * sizeof(__half), 256);
    a.part_o = (__half*)ws;
    a.part_ml = (float*)((char*)ws + o_bytes);
  }
  for (int i = 0; i < kApMaxRope / 2; ++i) a.freq[i] = i < g.rope_dim / 2 ? rope_freq(g.rope, i) : 0.0;
  CUtensorMap tq, to, tc, tr;
  CSA_CHECK(make_tmap_bf16(&tq, g.q, kApDim, (uint64_t)LB * g.Tq * kApHeads, 64, kApHeads));
  CSA_CHECK(make_tmap_bf16(&to, g.out, kApDim, (uint64_t)LB * g.Tq * kApHeads, 32, kApHeads,
                           CU_TENSOR_MAP_SWIZZLE_64B));
  // row gathers (one-row boxes of 64 dims); a cache with no rows is never
  // read, and its map is made over q instead
  const uint64_t n_cmp_rows = (uint64_t)g.B * g.n_max, n_raw_rows = (uint64_t)g.B * g.raw_max;
  const uint64_t n_q_rows = (uint64_t)g.B * g.Tq * kApHeads;
  if (kFp8) {  // E4M3 codes: one-row boxes of 128 dims (128 B)
    CSA_CHECK(make_tmap_u8(&tc, n_cmp_rows ? g.kv_cmp : g.q, kApDim,
                           n_cmp_rows ? n_cmp_rows : n_q_rows, 128));
    CSA_CHECK(make_tmap_u8(&tr, n_raw_rows ? g.kv_raw : g.q, kApDim,
                           n_raw_rows ? n_raw_rows : n_q_rows, 128));
  } else {
    CSA_CHECK(make_tmap_bf16(&tc, n_cmp_rows ? g.kv_cmp : g.q, kApDim,
                             n_cmp_rows ? n_cmp_rows : n_q_rows, 64, 1));
    CSA_CHECK(make_tmap_bf16(&tr, n_raw_rows ? g.kv_raw : g.q, kApDim,
                             n_raw_rows ? n_raw_rows : n_q_rows, 64, 1));
  }
  CSA_CHECK(set_smem_attr(k_attn_pair<kHca, kFp8>, kApSmemBytes, "k_attn_pair"));
  dim3 grid((unsigned)(2 * sp), (unsigned)(LB * g.Tq));
  cudaError_t e = launch_ex(k_attn_pair<kHca, kFp8>, grid,
                            dim3(kFp8 ? kApThreadsFp8 : kApThreads), kApSmemBytes, s, 2, a, tq, to,
                            tc, tr);
  if (e != cudaSuccess) return cuda_fail(e, "k_attn_pair");
  CSA_CHECK(launched("k_attn_pair"));
  if (sp == 1) return CSA_OK;
  AttnMergeArgs m;
  m.part_o = a.part_o;
  m.part_ml = a.part_ml;
  m.sink = g.sink;
  m.q_pos = g.q_pos;
  m.splits = sp;
  m.rope_dim = g.rope_dim;
  m.rows_per_layer = g.B * g.Tq;
  m.out = a.out;
  for (int i = 0; i < kApMaxRope / 2; ++i) m.freq[i] = a.freq[i];
  e = launch_ex(k_attn_merge, dim3(2 * kApSlabs, (unsigned)(LB * g.Tq)), dim3(kApHeads), 0, s, 1,
                m);
  if (e != cudaSuccess) return cuda_fail(e, "k_attn_merge");
  return launched("k_attn_merge");
}

static AttnArgs make_attn_args(const csa_params_t* p, const void* q, const int32_t* q_pos,
                               const void* kv_cmp, const int32_t* idx, const int32_t* n_cmp,
                               int32_t n_max, const void* kv_raw, const int32_t* raw_pos0,
                               const int32_t* n_raw, int32_t raw_max, const float* sink,
                               int32_t B, int32_t Tq, void* out) {
  AttnArgs a;
  a.q = q; a.q_pos = q_pos; a.kv_cmp = kv_cmp; a.idx = idx; a.n_cmp = n_cmp; a.n_max = n_max;
  a.kv_raw = kv_raw; a.raw_pos0 = raw_pos0; a.n_raw = n_raw; a.raw_max = raw_max; a.sink = sink;
  a.cmp_scale = nullptr; a.raw_scale = nullptr; a.layers = 1;
  a.B = B; a.Tq = Tq; a.H = p->n_heads; a.d = p->d; a.rope_dim = p->rope_dim; a.topk = p->topk;
  a.window = p->window; a.width = p->width; a.stride = p->stride; a.scale = attn_scale(p);
  a.rope = rope_spec(p); a.out = out;
  return a;
}

CSA_API csa_status_t csa_sparse_attn(const csa_params_t* p, csa_dtype_t dtype, const void* q,
                             const int32_t* q_pos, const void* kv_cmp, const int32_t* idx,
                             int32_t n_max, const void* kv_raw, const int32_t* raw_pos0,
                             const int32_t* n_raw, int32_t raw_max, const float* sink,
                             int32_t B, int32_t Tq, void* out, void* ws, size_t ws_bytes,
                             void* stream) {
  const CallRange trace("csa_sparse_attn");
  CSA_CHECK(attn_common_checks(p, dtype, q, q_pos, kv_cmp, n_max, kv_raw, raw_pos0, n_raw,
                               raw_max, sink, B, Tq, out));
  CSA_CHECK(check_topk(p));
  CSA_CHECK(check_ptr(idx, "idx"));
  CSA_CHECK(check_device());
  AttnArgs a = make_attn_args(p, q, q_pos, kv_cmp, idx, nullptr, n_max, kv_raw, raw_pos0, n_raw,
                              raw_max, sink, B, Tq, out);
  if (attn_tc_ok(p, dtype, false, n_max))
    return launch_attn_tc<false>(p, a, ws, ws_bytes, (cudaStream_t)stream);
  return launch_attn_simt<false>(a, dtype, (cudaStream_t)stream);
}

CSA_API csa_status_t csa_reuse_attn(const csa_params_t* p, csa_dtype_t dtype, int32_t layers,
                                    const void* q, const int32_t* q_pos, const void* kv_cmp,
                                    const int32_t* idx, int32_t n_max, const void* kv_raw,
                                    const int32_t* raw_pos0, const int32_t* n_raw,
                                    int32_t raw_max, const float* sink, int32_t B, int32_t Tq,
                                    void* out, void* ws, size_t ws_bytes, void* stream) {
  const CallRange trace("csa_reuse_attn");
  CSA_CHECK(attn_common_checks(p, dtype, q, q_pos, kv_cmp, n_max, kv_raw, raw_pos0, n_raw,
                               raw_max, sink, B, Tq, out));
  CSA_CHECK(check_topk(p));
  CSA_CHECK(check_ptr(idx, "idx"));
  if (layers < 1 || (long long)layers * B * Tq > 65535)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "layers=%d x B*Tq=%d beyond 65535 query rows", layers,
                B * Tq);
  CSA_CHECK(check_device());
  AttnArgs a = make_attn_args(p, q, q_pos, kv_cmp, idx, nullptr, n_max, kv_raw, raw_pos0, n_raw,
                              raw_max, sink, B, Tq, out);
  cudaStream_t s = (cudaStream_t)stream;
  if (attn_tc_ok(p, dtype, false, n_max)) {
    a.layers = layers;
    return launch_attn_tc<false>(p, a, ws, ws_bytes, s);
  }
  // generic path: one launch per layer
  const size_t esz = dtype == CSA_BF16 ? 2 : 4;
  const size_t per = (size_t)B * Tq * p->n_heads * p->d * esz;
  for (int r = 0; r < layers; ++r) {
    AttnArgs ar = a;
    ar.q = (const char*)q + r * per;
    ar.out = (char*)out + r * per;
    ar.sink = sink + (size_t)r * p->n_heads;
    CSA_CHECK(launch_attn_simt<false>(ar, dtype, s));
  }
  return CSA_OK;
}

CSA_API csa_status_t hca_attn(const csa_params_t* p, csa_dtype_t dtype, const void* q,
                      const int32_t* q_pos, const void* kv_cmp, const int32_t* n_cmp,
                      int32_t n_max, const void* kv_raw, const int32_t* raw_pos0,
                      const int32_t* n_raw, int32_t raw_max, const float* sink, int32_t B,
                      int32_t Tq, void* out, void* ws, size_t ws_bytes, void* stream) {
  const CallRange trace("hca_attn");
  CSA_CHECK(attn_common_checks(p, dtype, q, q_pos, kv_cmp, n_max, kv_raw, raw_pos0, n_raw,
                               raw_max, sink, B, Tq, out));
  CSA_CHECK(check_ptr(n_cmp, "n_cmp"));
  CSA_CHECK(check_device());
  AttnArgs a = make_attn_args(p, q, q_pos, kv_cmp, nullptr, n_cmp, n_max, kv_raw, raw_pos0,
                              n_raw, raw_max, sink, B, Tq, out);
  if (attn_tc_ok(p, dtype, true, n_max))
    return launch_attn_tc<true>(p, a, ws, ws_bytes, (cudaStream_t)stream);
  return launch_attn_simt<true>(a, dtype, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// FP8 KV cache (quantized after RoPE): quantizer and the attention calls
// over E4M3 caches.
// ---------------------------------------------------------------------------
CSA_API csa_status_t csa_quantize_fp8(csa_dtype_t dtype, const void* rows, int64_t n, int32_t d,
                                      uint8_t* codes, float* scales, void* stream) {
  const CallRange trace("csa_quantize_fp8");
  CSA_CHECK(check_dtype(dtype));
  if (n < 0 || d < 8 || d > 1024 || (d & 31))
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "n=%lld d=%d: d a multiple of 32 in [32, 1024]",
                (long long)n, d);
  if (n == 0) return CSA_OK;
  CSA_CHECK(check_ptr(rows, "rows"));
  CSA_CHECK(check_ptr(codes, "codes"));
  CSA_CHECK(check_ptr(scales, "scales"));
  CSA_CHECK(check_device());
  const long long ctas = (n + kQuantWarps - 1) / kQuantWarps;
  if (ctas > 2147483647LL) return fail(CSA_ERR_UNSUPPORTED_SHAPE, "n=%lld", (long long)n);
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == CSA_BF16)
    k_quantize_fp8<__nv_bfloat16><<<(unsigned)ctas, 32 * kQuantWarps, 0, s>>>(
        (const __nv_bfloat16*)rows, n, d, codes, scales);
  else
    k_quantize_fp8<float><<<(unsigned)ctas, 32 * kQuantWarps, 0, s>>>((const float*)rows, n, d,
                                                                      codes, scales);
  return launched("k_quantize_fp8");
}

static csa_status_t attn_fp8_checks(const csa_params_t* p, bool hca, const void* q,
                                    const int32_t* q_pos, const void* kv_cmp,
                                    const float* cmp_scale, int32_t n_max, const void* kv_raw,
                                    const float* raw_scale, const int32_t* raw_pos0,
                                    const int32_t* n_raw, int32_t raw_max, const float* sink,
                                    int32_t B, int32_t Tq, void* out) {
  CSA_CHECK(attn_common_checks(p, CSA_BF16, q, q_pos, kv_cmp, n_max, kv_raw, raw_pos0, n_raw,
                               raw_max, sink, B, Tq, out));
  CSA_CHECK(check_ptr(cmp_scale, "cmp_scale", n_max == 0));
  CSA_CHECK(check_ptr(raw_scale, "raw_scale", raw_max == 0));
  if (!attn_tc_ok(p, CSA_BF16, hca, n_max))
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "FP8 caches take the tensor-core path only: d = 512, 128 heads, rope_dim <= %d, "
                "at most %d rows per query", kApMaxRope, kApRowCap - 8);
  return CSA_OK;
}

CSA_API csa_status_t csa_sparse_attn_fp8(const csa_params_t* p, const void* q,
                                         const int32_t* q_pos, const uint8_t* kv_cmp,
                                         const float* cmp_scale, const int32_t* idx,
                                         int32_t n_max, const uint8_t* kv_raw,
                                         const float* raw_scale, const int32_t* raw_pos0,
                                         const int32_t* n_raw, int32_t raw_max, const float* sink,
                                         int32_t B, int32_t Tq, void* out, void* ws,
                                         size_t ws_bytes, void* stream) {
  const CallRange trace("csa_sparse_attn_fp8");
  CSA_CHECK(attn_fp8_checks(p, false, q, q_pos, kv_cmp, cmp_scale, n_max, kv_raw, raw_scale,
                            raw_pos0, n_raw, raw_max, sink, B, Tq, out));
  CSA_CHECK(check_topk(p));
  CSA_CHECK(check_ptr(idx, "idx"));
  CSA_CHECK(check_device());
  AttnArgs a = make_attn_args(p, q, q_pos, kv_cmp, idx, nullptr, n_max, kv_raw, raw_pos0, n_raw,
                              raw_max, sink, B, Tq, out);
  a.cmp_scale = cmp_scale;
  a.raw_scale = raw_scale;
  return launch_attn_tc<false, true>(p, a, ws, ws_bytes, (cudaStream_t)stream);
}

CSA_API csa_status_t hca_attn_fp8(const csa_params_t* p, const void* q, const int32_t* q_pos,
                                  const uint8_t* kv_cmp, const float* cmp_scale,
                                  const int32_t* n_cmp, int32_t n_max, const uint8_t* kv_raw,
                                  const float* raw_scale, const int32_t* raw_pos0,
                                  const int32_t* n_raw, int32_t raw_max, const float* sink,
                                  int32_t B, int32_t Tq, void* out, void* ws, size_t ws_bytes,
                                  void* stream) {
  const CallRange trace("hca_attn_fp8");
  CSA_CHECK(attn_fp8_checks(p, true, q, q_pos, kv_cmp, cmp_scale, n_max, kv_raw, raw_scale,
                            raw_pos0, n_raw, raw_max, sink, B, Tq, out));
  CSA_CHECK(check_ptr(n_cmp, "n_cmp"));
  CSA_CHECK(check_device());
  AttnArgs a = make_attn_args(p, q, q_pos, kv_cmp, nullptr, n_cmp, n_max, kv_raw, raw_pos0,
                              n_raw, raw_max, sink, B, Tq, out);
  a.cmp_scale = cmp_scale;
  a.raw_scale = raw_scale;
  return launch_attn_tc<true, true>(p, a, ws, ws_bytes, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// csa_index_topk_noalloc: the indexer + top-k for callers that cannot call
// cudaMalloc (or hand out a workspace).  The scores live in the fixed
// device array below instead of the caller's workspace.  Every GPU that
// loads this library keeps the array (8 MiB) until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScoreFloats = size_t(1) << 21;  // B * Tq * n_max limit
static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreFloats];

// Device address of g_noalloc_scores in the current context.  In host code
// the symbol's name is only a host-side stand-in, so the address is looked
// up with cudaGetSymbolAddress on the first call in a context and cached
// under that context's unique id (a reset device or another context on the
// same device loads the module again, possibly elsewhere, and gets its own
// entry).
using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

static csa_status_t current_context_id(unsigned long long* id) {
  static PfnCtxGetCurrent get_current = nullptr;
  static PfnCtxGetId get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* p1 = nullptr;
    void* p2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      return fail(CSA_ERR_CUDA, "driver entry points cuCtxGetCurrent / cuCtxGetId unavailable");
    get_current = reinterpret_cast<PfnCtxGetCurrent>(p1);
    get_id = reinterpret_cast<PfnCtxGetId>(p2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return fail(CSA_ERR_CUDA, "no current CUDA context");
  if (get_id(ctx, id) != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "cuCtxGetId failed");
  return CSA_OK;
}

static csa_status_t noalloc_scores_ptr(float** out) {
  struct Entry {
    unsigned long long ctx;
    float* ptr;
  };
  static Entry cache[64];
  static int n_cache = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx) == CSA_OK;
  if (have_ctx)
    for (int i = 0; i < n_cache; ++i)
      if (cache[i].ctx == ctx) {
        *out = cache[i].ptr;
        return CSA_OK;
      }
  // first call in this context (or none is current yet: the runtime makes
  // the device's primary context current here)
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scores);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
  if (!have_ctx) CSA_CHECK(current_context_id(&ctx));
  cache[n_cache < 64 ? n_cache++ : 63] = Entry{ctx, static_cast<float*>(p)};
  *out = static_cast<float*>(p);
  return CSA_OK;
}

CSA_API csa_status_t csa_index_topk_noalloc(const csa_params_t* p, csa_dtype_t dtype,
                                            const void* q_idx, const float* w, const void* k_idx,
                                            const int32_t* q_pos, const int32_t* n_cmp,
                                            int32_t B, int32_t Tq, int32_t n_max,
                                            int32_t* idx_out, void* stream) {
  const CallRange trace("csa_index_topk_noalloc");
  CSA_CHECK(check_params(p));
  CSA_CHECK(check_dtype(dtype));
  CSA_CHECK(check_indexer_shape(p));
  CSA_CHECK(check_topk(p));
  CSA_CHECK(check_sizes(B, Tq, n_max));
  CSA_CHECK(check_ptr(q_idx, "q_idx"));
  CSA_CHECK(check_ptr(w, "w"));
  CSA_CHECK(check_ptr(k_idx, "k_idx", n_max == 0));
  CSA_CHECK(check_ptr(q_pos, "q_pos"));
  CSA_CHECK(check_ptr(n_cmp, "n_cmp"));
  CSA_CHECK(check_ptr(idx_out, "idx_out"));
  // scores first, then the top-k candidate lists of long rows
  const size_t sb = scores_bytes(B, Tq, n_max);
  const size_t tb = topk_ws_bytes(p, B, Tq, n_max);
  if (sb + tb > kNoAllocScoreFloats * sizeof(float))
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "scores (%zu bytes) and top-k candidate lists (%zu bytes) exceed the no-alloc "
                "scratch of %zu bytes; use csa_index_topk with a workspace",
                sb, tb, kNoAllocScoreFloats * sizeof(float));
  CSA_CHECK(check_device());
  float* scores = nullptr;
  CSA_CHECK(noalloc_scores_ptr(&scores));
  cudaStream_t s = (cudaStream_t)stream;
  CSA_CHECK(index_scores_impl(p, dtype, q_idx, w, k_idx, q_pos, n_cmp, B, Tq, n_max, scores, s));
  return topk_impl(p, scores, q_pos, n_cmp, B, Tq, n_max, idx_out, (char*)scores + sb,
                   kNoAllocScoreFloats * sizeof(float) - sb, s);
}

static std::atomic<int32_t> g_last_site{0};

CSA_API csa_status_t csa_poll_device_error(void* stream) {
  const CallRange trace("csa_poll_device_error");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0, site = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (v == 0) return CSA_OK;
  e = cudaMemcpyFromSymbol(&site, g_device_error_site, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error site");
  g_last_site.store(site, std::memory_order_relaxed);
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error_site, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  return fail((csa_status_t)v, "device reported %s (kernel source line %d)",
              csa_status_string((csa_status_t)v), site);
}

CSA_API int32_t csa_last_device_error_site(void) {
  return g_last_site.load(std::memory_order_relaxed);
}

