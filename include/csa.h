/*
 * csa.h - C ABI of the B200 (sm_100a) Compressed Sparse Attention library.
 *
 * The layer (DeepSeek-V4 style), as stated on "DeepSeek-V4-Pro vs Inkling"
 * (archdiff.com/compare/deepseek-v4-vs-inkling), component table:
 *   - row "Compressed Sparse Attention": each KV entry pools 8 overlapping
 *     tokens at stride m = 4 with a per-channel softmax; a lightning indexer
 *     (64 heads x 128 dims, ReLU scores weighted per head) keeps the top
 *     1,024 entries; the 128 query heads attend to them together with the
 *     sliding-window (SWA) entries;
 *   - row "Heavily Compressed Attention": every 128 tokens pooled into one
 *     entry, dense shared-KV attention over all of them plus a 128-token
 *     window;
 *   - row "Partial RoPE": RoPE on the last 64 of 512 dims of queries and KV
 *     entries; each entry is both key and value, so the same 64 dims of
 *     every head's output are rotated by -i (inverse rotation at the query
 *     position);
 *   - row "Output gate + sink": per-head learnable sink logit whose
 *     exponential is added to the softmax denominator.
 * Shapes: "DeepSeek-V4-Pro" fact sheet (llm-atlas), raw config fields
 * (head_dim 512, qk_rope_head_dim 64, num_attention_heads 128,
 * num_key_value_heads 1, index_n_heads 64, index_head_dim 128,
 * index_topk 1024, sliding_window 128, rope_theta 10000).
 *
 * Conventions shared by every call
 * ---------------------------------
 * Ownership: every data pointer is a DEVICE pointer owned by the caller.
 *   The library never allocates device memory; scratch space, where a call
 *   needs it, is the caller's `ws` buffer of at least csa_workspace_size()
 *   bytes.  `stream` is a cudaStream_t (NULL = legacy default stream).
 * Layout: dense row-major arrays, innermost dimension last.  Every array's
 *   base address must be 16-byte aligned (CSA_ERR_MISALIGNED otherwise).
 *   Element type of the "value" arrays (x, gate, q, kv caches, indexer
 *   q/k, out) is the call's csa_dtype_t; weights, sink and scores are fp32;
 *   positions, counts and indices are int32.
 * Sizes: B >= 1 sequences of Tq >= 1 query tokens with B * Tq <= 65535, and
 *   n_max >= 0 entries per sequence; otherwise CSA_ERR_UNSUPPORTED_SHAPE.
 * Positions: token t of a sequence sits at position t (the first token at
 *   0).  Entry j pools tokens stride*j .. stride*j + width - 1 and is rotated
 *   at position stride*j + pos_offset.  Entry j is visible to a query at
 *   position t iff j < n_cmp and stride*j + width - 1 <= t.  The window of a
 *   query at t is the raw rows of tokens max(0, t-window+1) .. t that the raw
 *   buffer holds (tokens raw_pos0 .. raw_pos0 + n_raw - 1).  KV caches hold
 *   RoPE-rotated rows.
 * Errors: host-side validation is synchronous and returns a status; no
 *   exception crosses the ABI.  Launch failures return CSA_ERR_CUDA (details
 *   from csa_last_error_detail(), per host thread).  Errors detected inside a
 *   kernel (a bounded wait that ran out) are recorded in a per-device error
 *   word that csa_poll_device_error() reads and clears.
 * Asynchrony: every compute call only enqueues work on `stream`; calls on
 *   different streams are independent.  The tensor-core kernels launch with
 *   programmatic dependent launch: one may start while its predecessor on
 *   the stream is finishing, but it waits for that predecessor to complete
 *   (and its writes to be visible) before its first access to global
 *   memory, so stream order holds for all data.  The attention calls with
 *   few query tokens launch thread-block clusters.
 * Tracing: every call that validates, sizes or launches (all but the plain
 *   getters and setters) is an NVTX v3 range in the domain "csa", named
 *   after the call and open for its host-side duration, early rejections
 *   included.  Without a tool attached (Nsight Systems, or a library named
 *   by NVTX_INJECTION64_PATH) a range costs one branch.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA_ABI_VERSION 2

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARGUMENT = 1,   /* null pointer, negative size, bad enum */
  CSA_ERR_MISALIGNED = 2,         /* a base address is not 16-byte aligned */
  CSA_ERR_UNSUPPORTED_SHAPE = 3,  /* a size outside the supported limits */
  CSA_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 */
  CSA_ERR_WORKSPACE_TOO_SMALL = 5,
  CSA_ERR_CUDA = 6,               /* a CUDA runtime call failed */
  CSA_ERR_DEVICE_TIMEOUT = 7,     /* a bounded device-side wait ran out */
  CSA_ERR_DEVICE_BOUNDS = 8       /* a device-side index check failed */
} csa_status_t;

typedef enum { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype_t;

typedef enum {
  CSA_OP_COMPRESS = 0,
  CSA_OP_INDEX_TOPK = 1,
  CSA_OP_SPARSE_ATTN = 2,
  CSA_OP_HCA_ATTN = 3,
  CSA_OP_TOPK_SELECT = 4
} csa_op_t;

/* Layer constants.  Defaults of the measured model: d 512, rope_dim 64,
 * theta 1e4, scale 1/sqrt(512), n_heads 128, idx_heads 64, idx_dim 128,
 * topk 1024, window 128, (width, stride) = (8, 4) for CSA and (128, 128)
 * for HCA, pos_offset 0, rope_factor 1 (plain RoPE).
 *
 * Extended RoPE ("DeepSeek-V4-Pro vs Inkling", "Partial RoPE" row: the
 * compressed layers use theta = 160,000 with YaRN, factor 16 over 65,536
 * tokens).  With rope_factor s > 1 every rotation of the call (queries,
 * entries, window rows, the output's inverse rotation) uses the YaRN
 * frequencies of Peng et al. 2023 ("YaRN: Efficient Context Window
 * Extension of Large Language Models", section 3): rotary pair i with
 * f_i = theta^(-2i/rope_dim) turns n_i = rope_orig_ctx * f_i / (2 pi) times
 * over the original context; with g = clamp((n_i - rope_beta_slow) /
 * (rope_beta_fast - rope_beta_slow), 0, 1) it rotates at (1 - g) f_i / s +
 * g f_i.  The attention calls then multiply `scale` by YaRN's temperature
 * (0.1 ln s + 1)^2.  The paper's beta values are 32 (fast) and 1 (slow). */
typedef struct {
  int32_t d;          /* entry / head dim, multiple of 32, <= 1024 */
  int32_t rope_dim;   /* rotated trailing dims, even, <= d (0 = no RoPE) */
  float theta;        /* RoPE base */
  float scale;        /* softmax scale on q.k (the sink logit is unscaled) */
  int32_t n_heads;    /* query heads H sharing one KV row (MQA) */
  int32_t idx_heads;  /* indexer heads H_I */
  int32_t idx_dim;    /* indexer dim d_I */
  int32_t topk;       /* k: entries kept per query */
  int32_t window;     /* W: raw window length */
  int32_t width;      /* pooling width w_c */
  int32_t stride;     /* pooling stride m */
  int32_t pos_offset; /* RoPE position of entry j is stride*j + pos_offset */
  float rope_factor;    /* YaRN factor s (<= 1: plain RoPE, the fields below unused) */
  int32_t rope_orig_ctx;  /* YaRN original context length L (>= 1 when s > 1) */
  float rope_beta_fast; /* YaRN beta: pairs turning more often over L keep f_i */
  float rope_beta_slow; /* YaRN alpha: pairs turning less often over L get f_i / s */
} csa_params_t;

/* Library ABI version (CSA_ABI_VERSION). */
int csa_abi_version(void);

/* Static text for a status code. */
const char* csa_status_string(csa_status_t status);

/* Text of the last non-OK status returned on this host thread. */
const char* csa_last_error_detail(void);

/* Bytes of caller workspace `op` needs for B sequences of Tq query tokens
 * over caches of n_max entries.  0 means the call needs none (ws may be
 * NULL). */
csa_status_t csa_workspace_size(const csa_params_t* p, csa_op_t op, int32_t B, int32_t Tq,
                                int32_t n_max, size_t* bytes);

/* Step 1 - compression ("Compressed Sparse Attention" row: pool 8 overlapping
 * tokens at stride 4 with a per-channel softmax; "Heavily Compressed
 * Attention" row with width = stride = 128).
 *   x, gate        [B][T][d]  token KV rows and per-channel gate logits
 *   kv_cmp_out     [B][N][d]  N = floor((T - width)/stride) + 1 pooled,
 *                  rotated entries:
 *                  e_j[c] = sum_u softmax_u(gate[s*j+u][c]) * x[s*j+u][c],
 *                  then RoPE at position s*j + pos_offset
 *   kv_raw_rot_out [B][T][d]  (nullable) x rotated at each token's position
 * Math in fp32; outputs rounded to the dtype (bf16: round to nearest even). */
csa_status_t csa_compress(const csa_params_t* p, csa_dtype_t dtype, const void* x,
                          const void* gate, int32_t B, int32_t T, void* kv_cmp_out,
                          void* kv_raw_rot_out, void* stream);

/* Step 1 during decode - incremental compression: the entries and rotated
 * raw rows that the tokens t_old[b] .. t_new[b] - 1 of each sequence
 * complete, appended to caller-owned caches ("Compressed Sparse Attention"
 * row: an entry pools tokens s*j .. s*j + width - 1, so it exists once token
 * s*j + width - 1 has arrived; "Heavily Compressed Attention" row: one entry
 * per 128 tokens).  Each written value equals what csa_compress writes for
 * the same tokens.
 *   x, gate   [B][L][d]  token rows; row i of sequence b is token x_pos0[b] + i
 *             (a window of the sequence that holds every token the new
 *             entries pool: from s * n_old back, n_old = entries before
 *             t_old[b], up to t_new[b] - 1)
 *   x_pos0, t_old, t_new  [B] int32, device; 0 <= t_new[b] - t_old[b] <= max_new
 *   kv_cmp    [B][n_cap][d]  entry j at row j; rows n_entries(t_old[b]) ..
 *             n_entries(t_new[b]) - 1 are written, n_entries(t) =
 *             floor((t - width)/s) + 1 for t >= width, else 0
 *   kv_raw    [B][raw_cap][d] (nullable): token t's rotated row at row
 *             t - raw_pos0[b], for t in t_old[b] .. t_new[b] - 1
 * max_new (host) bounds the tokens any sequence adds and sizes the launch.
 * Rows outside these ranges are left untouched.  A sequence whose range
 * breaks these rules (t_new < t_old, more than max_new tokens) is skipped
 * whole, a row that needs a token outside x or lands outside its cache is
 * skipped; both record CSA_ERR_DEVICE_BOUNDS (csa_poll_device_error). */
csa_status_t csa_compress_append(const csa_params_t* p, csa_dtype_t dtype, const void* x,
                                 const void* gate, const int32_t* x_pos0, int32_t B, int32_t L,
                                 const int32_t* t_old, const int32_t* t_new, int32_t max_new,
                                 void* kv_cmp, int32_t n_cap, void* kv_raw,
                                 const int32_t* raw_pos0, int32_t raw_cap, void* stream);

/* Step 2a - lightning indexer scores ("64 heads x 128 dims, ReLU scores
 * weighted per head").
 *   q_idx  [B][Tq][H_I][d_I], w [B][Tq][H_I] fp32, k_idx [B][n_max][d_I]
 *   q_pos  [B][Tq] int32, n_cmp [B] int32 (valid entries, <= n_max)
 *   scores [B][Tq][n_max] fp32: scores[b][t][j] =
 *          sum_h w[b][t][h] * max(0, q_idx[b][t][h] . k_idx[b][j]) for every
 *          visible j; entries j >= n_visible are not written.
 * fp32 products and sums: exact whenever the inputs are integers and powers
 * of two small enough that every partial sum fits in 24 bits. */
csa_status_t csa_index_scores(const csa_params_t* p, csa_dtype_t dtype, const void* q_idx,
                              const float* w, const void* k_idx, const int32_t* q_pos,
                              const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                              float* scores, void* stream);

/* Step 2b - top-k ("keeps the top 1,024 entries") on given scores.
 *   scores  [B][Tq][n_max] fp32 (only visible entries are read)
 *   idx_out [B][Tq][topk] int32: the topk largest visible scores, ties to
 *           the lower index, in ascending index order, padded with -1; all
 *           visible entries when there are at most topk.  -0.0 == +0.0.
 *           NaN scores give an unspecified (but valid) selection.
 *   ws      csa_workspace_size(CSA_OP_TOPK_SELECT) bytes. */
csa_status_t csa_topk_select(const csa_params_t* p, const float* scores, const int32_t* q_pos,
                             const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                             int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/* Step 2 - indexer + top-k in one call (scores kept in `ws`).  Arguments as
 * csa_index_scores / csa_topk_select; ws of csa_workspace_size(
 * CSA_OP_INDEX_TOPK) bytes. */
csa_status_t csa_index_topk(const csa_params_t* p, csa_dtype_t dtype, const void* q_idx,
                            const float* w, const void* k_idx, const int32_t* q_pos,
                            const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                            int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/* Step 3 - sparse shared-KV MQA ("the 128 query heads attend to [the
 * selected entries] together with the SWA entries"; sink and partial RoPE
 * as above).
 *   q        [B][Tq][H][d] unrotated queries; q_pos [B][Tq]
 *   kv_cmp   [B][n_max][d] rotated entries; idx [B][Tq][topk] (-1 = unused)
 *   kv_raw   [B][raw_max][d] rotated raw rows of tokens raw_pos0[b] ..
 *            raw_pos0[b] + n_raw[b] - 1 (n_raw[b] <= raw_max)
 *   sink     [H] fp32
 *   out      [B][Tq][H][d]: per head h, with q^ = RoPE(q, t) and rows r_i
 *            the selected entries then the window rows:
 *            z_i = scale * q^.r_i,  a_i = exp(z_i) / (exp(sink_h) + sum exp z),
 *            o = sum_i a_i r_i, then dims d-rope_dim.. rotated at -t.
 * bf16: q^ and the softmax weights are rounded to bf16 for the tensor-core
 * products, accumulation is fp32.  ws: csa_workspace_size(CSA_OP_SPARSE_ATTN). */
csa_status_t csa_sparse_attn(const csa_params_t* p, csa_dtype_t dtype, const void* q,
                             const int32_t* q_pos, const void* kv_cmp, const int32_t* idx,
                             int32_t n_max, const void* kv_raw, const int32_t* raw_pos0,
                             const int32_t* n_raw, int32_t raw_max, const float* sink,
                             int32_t B, int32_t Tq, void* out, void* ws, size_t ws_bytes,
                             void* stream);

/* CSA2 Reuse layers ("DeepSeek-V4.1-Flash vs Inkling", row "CSA2 encoder
 * layers (2x compression, Full + Reuse)": the KV is computed in 3 of 18
 * layers, the rest reuse that KV and its top-512 selection): csa_sparse_attn
 * for `layers` layers at once, each with its own queries, sink and output,
 * all over the same entries, selection and window.
 *   q    [layers][B][Tq][H][d], sink [layers][H], out [layers][B][Tq][H][d]
 *   q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw: as csa_sparse_attn (shared)
 * layers * B * Tq <= 65535 (CSA_ERR_UNSUPPORTED_SHAPE otherwise).
 * ws: csa_workspace_size(CSA_OP_SPARSE_ATTN, layers * B, Tq, n_max). */
csa_status_t csa_reuse_attn(const csa_params_t* p, csa_dtype_t dtype, int32_t layers,
                            const void* q, const int32_t* q_pos, const void* kv_cmp,
                            const int32_t* idx, int32_t n_max, const void* kv_raw,
                            const int32_t* raw_pos0, const int32_t* n_raw, int32_t raw_max,
                            const float* sink, int32_t B, int32_t Tq, void* out, void* ws,
                            size_t ws_bytes, void* stream);

/* Step 4 - HCA dense shared-KV attention ("dense shared-KV attention over all
 * of them plus a 128-token window"): as csa_sparse_attn with the selected
 * set replaced by every visible entry j < n_cmp[b] (p->width, p->stride give
 * visibility).  ws: csa_workspace_size(CSA_OP_HCA_ATTN). */
csa_status_t hca_attn(const csa_params_t* p, csa_dtype_t dtype, const void* q,
                      const int32_t* q_pos, const void* kv_cmp, const int32_t* n_cmp,
                      int32_t n_max, const void* kv_raw, const int32_t* raw_pos0,
                      const int32_t* n_raw, int32_t raw_max, const float* sink, int32_t B,
                      int32_t Tq, void* out, void* ws, size_t ws_bytes, void* stream);

/* KV cache quantized after RoPE ("DeepSeek-V4.1-Flash vs Inkling", "Partial
 * RoPE" row: the KV cache is quantized after RoPE; the pages give no
 * format).  Format of this library: OCP 8-bit float E4M3 codes (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits, no infinities, largest finite
 * 448) with one fp32 scale per cache row.
 *   rows   [n][d] (dtype bf16 or fp32) rotated cache rows, d a multiple of 32
 *          in [32, 1024]
 *   codes  [n][d] uint8: code = x / scale rounded to the nearest E4M3 value
 *          (ties to even), saturated at +-448
 *   scales [n] fp32: scale = max|row| / 448, 1 for an all-zero row
 * The scale and the division are IEEE fp32 (correctly rounded). */
csa_status_t csa_quantize_fp8(csa_dtype_t dtype, const void* rows, int64_t n, int32_t d,
                              uint8_t* codes, float* scales, void* stream);

/* Steps 3/4 over FP8 caches: csa_sparse_attn and hca_attn with kv_cmp
 * [B][n_max][d] and kv_raw [B][raw_max][d] holding E4M3 codes and
 * cmp_scale [B][n_max], raw_scale [B][raw_max] their row scales (as
 * csa_quantize_fp8 writes them).  A row stands for code value x scale; the
 * kernel rounds that product to bf16 once before the products.  q and out
 * are bf16; the tensor-core shape only (d = 512, 128 heads, rope_dim <= 128,
 * topk (or n_max) + window + 8 <= 2048 rows), CSA_ERR_UNSUPPORTED_SHAPE
 * otherwise.  ws: csa_workspace_size(CSA_OP_SPARSE_ATTN / CSA_OP_HCA_ATTN). */
csa_status_t csa_sparse_attn_fp8(const csa_params_t* p, const void* q, const int32_t* q_pos,
                                 const uint8_t* kv_cmp, const float* cmp_scale,
                                 const int32_t* idx, int32_t n_max, const uint8_t* kv_raw,
                                 const float* raw_scale, const int32_t* raw_pos0,
                                 const int32_t* n_raw, int32_t raw_max, const float* sink,
                                 int32_t B, int32_t Tq, void* out, void* ws, size_t ws_bytes,
                                 void* stream);
csa_status_t hca_attn_fp8(const csa_params_t* p, const void* q, const int32_t* q_pos,
                          const uint8_t* kv_cmp, const float* cmp_scale, const int32_t* n_cmp,
                          int32_t n_max, const uint8_t* kv_raw, const float* raw_scale,
                          const int32_t* raw_pos0, const int32_t* n_raw, int32_t raw_max,
                          const float* sink, int32_t B, int32_t Tq, void* out, void* ws,
                          size_t ws_bytes, void* stream);

/* Indexer + top-k that allocates nothing: the same computation and
 * arguments as csa_index_topk, without `ws`.  The pages have no counterpart
 * of this call; it serves callers that cannot call cudaMalloc or hand out a
 * workspace - a host that passes the library only its input and output
 * buffers, an engine whose allocator has already reserved all device
 * memory, or a latency-critical loop that cannot afford cudaMalloc's
 * device-wide synchronization.
 *   Scratch: a fixed 8 MiB array compiled into the library; every GPU that
 *   loads the library holds it until the process exits.  It holds the
 *   scores (B * Tq * n_max fp32, rounded up to 256 bytes) and, for rows too
 *   long for one top-k block, the per-chunk candidate lists: the call needs
 *   csa_workspace_size(CSA_OP_INDEX_TOPK) <= 8 MiB (so at most 2^21 scores)
 *   and returns CSA_ERR_UNSUPPORTED_SHAPE beyond that.  Nothing in the array
 *   needs clearing: each call writes everything it reads.
 *   The first call in a CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress) and caches it under that context's id (a reset
 *   device, or another context made current on the same device, looks it up
 *   again); make that first call before any stream capture.
 *   Every call shares the one array: calls whose work overlaps on the GPU
 *   (different streams, or other host threads) race and give wrong indices.
 *   Serialize them. */
csa_status_t csa_index_topk_noalloc(const csa_params_t* p, csa_dtype_t dtype, const void* q_idx,
                                    const float* w, const void* k_idx, const int32_t* q_pos,
                                    const int32_t* n_cmp, int32_t B, int32_t Tq, int32_t n_max,
                                    int32_t* idx_out, void* stream);

/* Limit, in nanoseconds, of every bounded wait inside the library's kernels
 * (a wait on a copy, an MMA or a cooperating CTA).  A wait that runs out
 * records CSA_ERR_DEVICE_TIMEOUT (read with csa_poll_device_error) and its
 * kernel winds down without finishing its output.  0 restores the default
 * of 2 s.  Process-wide, read when a kernel is launched (a captured CUDA
 * graph keeps the limit it was captured with).  A diagnostic: a tiny limit
 * makes the timeout path run on purpose. */
void csa_set_wait_limit_ns(uint64_t ns);

/* Number of kernels this library has launched (or recorded into a stream
 * capture) in this process so far, on every device and host thread.  A
 * diagnostic: the difference across one call is that call's kernel count. */
uint64_t csa_launch_count(void);

/* Synchronizes `stream`, then reads and clears the current device's error
 * word: CSA_OK, CSA_ERR_DEVICE_TIMEOUT or CSA_ERR_DEVICE_BOUNDS. */
csa_status_t csa_poll_device_error(void* stream);

/* The source line, in the library's kernel sources, of the device-side check
 * that recorded the error the last failing csa_poll_device_error() returned
 * (in this process, on any device); 0 before any.  A diagnostic: for a
 * timeout it names the wait that ran out first. */
int32_t csa_last_device_error_site(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
