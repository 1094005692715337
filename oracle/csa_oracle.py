"""fp64 CPU oracle of the CSA / HCA attention layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
runs this module; only the tests, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` do.  It shares no code
with the CUDA path.

Plain NumPy in float64 on the exact input values (bf16 inputs are widened
exactly).  Every step follows the layer as the pages state it, in the pages'
order:

* "DeepSeek-V4-Pro vs Inkling" (archdiff.com/compare/deepseek-v4-vs-inkling),
  component table, row "Compressed Sparse Attention": each KV entry pools 8
  overlapping tokens at stride m = 4 with a per-channel softmax; a lightning
  indexer of 64 heads x 128 dims scores entries with per-head weighted ReLU
  dot products and keeps the top 1,024; the 128 query heads attend to those
  entries together with the sliding-window (SWA) entries.
* same table, row "Heavily Compressed Attention": every 128 tokens pool into
  one entry; dense shared-KV attention over all entries plus a 128-token
  window.
* same table, row "Partial RoPE": RoPE on the last 64 of 512 dims of queries
  and KV entries; each entry is both key and value, so the same 64 dims of
  every head's output are rotated by -i (the inverse rotation at the query's
  position).
* same table, row "Output gate + sink": a per-head learnable sink logit whose
  exponential joins the softmax denominator.
* "DeepSeek-V4-Pro" fact sheet (llm-atlas), raw config fields: head_dim 512,
  qk_rope_head_dim 64, rope_theta 10000, index_n_heads 64, index_head_dim 128,
  index_topk 1024, sliding_window 128, num_key_value_heads 1.

Readings of points the pages leave open:

* entry j pools tokens stride*j .. stride*j + width - 1, no padding, so
  N(T) = floor((T - width) / stride) + 1;
* gate logits g[t, c] are a layer input, one per token and channel;
* entry j sits at position stride*j + pos_offset for RoPE; raw window rows
  sit at their own token position;
* RoPE pairs are interleaved (d-r+2i, d-r+2i+1) with frequency
  theta**(-2i/r), rotated as a complex number times exp(i * pos * freq);
  where a layer extends it with YaRN (theta = 160,000, factor 16 over
  65,536 tokens), one YaRN spec serves q, entries, window rows and output;
* the softmax scale is 1/sqrt(d) on the whole q.k; the sink logit is not
  scaled;
* entry j is visible to the query at token t iff its last token
  stride*j + width - 1 <= t; the window is tokens t-W+1 .. t (clipped at 0);
* top-k keeps the k largest scores, ties to the lower index, returned in
  ascending index order and padded with -1; with fewer than k visible
  entries all are kept;
* no de-duplication between window rows and compressed entries;
* CSA2 ("DeepSeek-V4.1-Flash vs Inkling", row "CSA2 encoder layers (2x
  compression, Full + Reuse)": KV pooled 2 -> 1, computed in 3 of 18 layers,
  the rest reuse that KV and its top-512 selection): a Full layer is this
  layer with width = stride = 2 and k = 512; a Reuse layer is sparse_attn
  with its own queries (and sink) over the Full layer's entries and indices.

Parity unpinned by the pages (conventions fixed here and given to the GPU
path as parameters): entry position, RoPE pair layout, window inclusivity,
decode query position.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

NEG_INF = float("-inf")


# --------------------------------------------------------------------------
# Entry counts and visibility ("Compressed Sparse Attention" row: 8 tokens at
# stride 4; "Heavily Compressed Attention" row: 128 tokens per entry)
# --------------------------------------------------------------------------
def n_compressed(T: int, width: int, stride: int) -> int:
    """Number of entries pooled from T tokens (no padding)."""
    if T < width:
        return 0
    return (T - width) // stride + 1


def n_visible(t: int, n_cmp: int, width: int, stride: int) -> int:
    """Entries j < n_cmp whose last token stride*j + width - 1 is <= t."""
    if t < width - 1:
        return 0
    return int(min(n_cmp, (t - width + 1) // stride + 1))


def window_tokens(t: int, window: int, raw_pos0: int, n_raw: int) -> np.ndarray:
    """Token positions of the sliding window of query t that the raw buffer
    (tokens raw_pos0 .. raw_pos0 + n_raw - 1) holds: max(0, t-W+1) .. t."""
    lo = max(0, t - window + 1, raw_pos0)
    hi = min(t, raw_pos0 + n_raw - 1)
    if hi < lo:
        return np.zeros((0,), dtype=np.int64)
    return np.arange(lo, hi + 1, dtype=np.int64)


# --------------------------------------------------------------------------
# Extended RoPE of the compressed layers ("DeepSeek-V4-Pro vs Inkling" and
# "DeepSeek-V4.1-Flash vs Inkling", "Partial RoPE" rows: theta = 160,000
# with YaRN, factor 16 over 65,536 tokens; "DeepSeek-V4-Pro" fact sheet,
# raw config field compress_rope_theta 160000).  The pages give no YaRN
# formula; this follows the published definition (Peng, Quesnelle, Fan,
# Shippole 2023, "YaRN: Efficient Context Window Extension of Large Language
# Models", section 3): per rotary pair i with frequency f_i = theta**(-2i/r)
# and wavelength 2 pi / f_i, r_i = L / wavelength counts the rotations the
# pair makes over the original context L; with
#   gamma_i = clip((r_i - alpha) / (beta - alpha), 0, 1)
# the new frequency is (1 - gamma_i) f_i / s + gamma_i f_i (pairs that turn
# fewer than alpha times are interpolated by the factor s, pairs that turn
# more than beta times keep their frequency), and the softmax logits are
# multiplied by (0.1 ln s + 1)**2 (the paper's attention temperature).
# alpha = 1 and beta = 32 are the paper's values.
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class YaRN:
    theta: float            # RoPE base
    factor: float           # s, the context-extension factor
    orig_ctx: int           # L, the context the frequencies were made for
    beta_fast: float = 32.0  # beta: rotations over L above which f_i is kept
    beta_slow: float = 1.0   # alpha: rotations over L below which f_i / s is used


def rope_freqs(rope_dim: int, theta) -> np.ndarray:
    """Frequencies of the rope_dim / 2 rotary pairs: theta**(-2i/r), or their
    YaRN interpolation when `theta` is a YaRN spec with factor > 1."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    if not isinstance(theta, YaRN):
        return np.power(float(theta), -2.0 * i / rope_dim)
    f = np.power(float(theta.theta), -2.0 * i / rope_dim)
    if theta.factor <= 1.0:
        return f
    turns = theta.orig_ctx * f / (2.0 * math.pi)
    gamma = np.clip((turns - theta.beta_slow) / (theta.beta_fast - theta.beta_slow), 0.0, 1.0)
    return (1.0 - gamma) * f / theta.factor + gamma * f


def attention_temperature(theta) -> float:
    """Factor on the softmax logits: (0.1 ln s + 1)**2 under YaRN, else 1."""
    if isinstance(theta, YaRN) and theta.factor > 1.0:
        return (0.1 * math.log(theta.factor) + 1.0) ** 2
    return 1.0


# --------------------------------------------------------------------------
# Partial RoPE ("Partial RoPE" row: last 64 of 512 dims; output rotated by -i)
# --------------------------------------------------------------------------
def rope(x: np.ndarray, pos, rope_dim: int, theta) -> np.ndarray:
    """Rotate the trailing `rope_dim` dims of x[..., d] at position(s) `pos`.

    Pair i = dims (d - r + 2i, d - r + 2i + 1), angle pos * f_i with
    f_i = theta**(-2i/r) (or the YaRN frequencies, see rope_freqs);
    (a, b) -> (a cos - b sin, a sin + b cos).  `pos` broadcasts against
    x.shape[:-1].  A negative position gives the inverse rotation.
    """
    x = np.array(x, dtype=np.float64, copy=True)
    if rope_dim == 0:
        return x
    d = x.shape[-1]
    freq = rope_freqs(rope_dim, theta)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., d - rope_dim::2].copy()
    b = x[..., d - rope_dim + 1::2].copy()
    x[..., d - rope_dim::2] = a * c - b * s
    x[..., d - rope_dim + 1::2] = a * s + b * c
    return x


# --------------------------------------------------------------------------
# Step 1: compression ("Compressed Sparse Attention" row: pool 8 overlapping
# tokens at stride 4 with a per-channel softmax; HCA row: 128 tokens -> 1)
# --------------------------------------------------------------------------
def compress(x: np.ndarray, g: np.ndarray, width: int, stride: int,
             rope_dim: int, theta, pos_offset: int = 0) -> np.ndarray:
    """Pool x[T, d] into N entries with per-channel softmax weights over the
    `width` taps of each entry, then rotate entry j at stride*j + pos_offset."""
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    T, d = x.shape
    N = n_compressed(T, width, stride)
    out = np.zeros((N, d), dtype=np.float64)
    for j in range(N):
        taps = slice(stride * j, stride * j + width)
        gj = g[taps]
        e = np.exp(gj - gj.max(axis=0))
        a = e / e.sum(axis=0)
        out[j] = (a * x[taps]).sum(axis=0)
    pos = stride * np.arange(N, dtype=np.int64) + pos_offset
    return rope(out, pos, rope_dim, theta)


def rotate_raw(x: np.ndarray, pos0: int, rope_dim: int, theta) -> np.ndarray:
    """Raw (uncompressed) token rows rotated at their own positions."""
    x = np.asarray(x, dtype=np.float64)
    return rope(x, pos0 + np.arange(x.shape[0], dtype=np.int64), rope_dim, theta)


# --------------------------------------------------------------------------
# Step 1 during decode: the entries and raw rows that newly arrived tokens
# complete ("Compressed Sparse Attention" row: an entry pools tokens
# stride*j .. stride*j + width - 1, so it exists once its last token has
# arrived; "Heavily Compressed Attention" row: one entry per 128 tokens)
# --------------------------------------------------------------------------
def compress_append(x_win: np.ndarray, g_win: np.ndarray, x_pos0: int, t_old: int, t_new: int,
                    width: int, stride: int, rope_dim: int, theta, pos_offset: int = 0):
    """Tokens t_old .. t_new - 1 arrive; x_win[i], g_win[i] are token
    x_pos0 + i.  The new entries are j0 = N(t_old) .. N(t_new) - 1: the batch
    compression of the tokens from stride*j0 on, whose positions start at
    stride*j0.  Returns (j0, entries [N(t_new) - j0, d], raw rows of tokens
    t_old .. t_new - 1 rotated at their positions)."""
    x_win = np.asarray(x_win, dtype=np.float64)
    g_win = np.asarray(g_win, dtype=np.float64)
    j0 = n_compressed(t_old, width, stride)
    j1 = n_compressed(t_new, width, stride)
    lo = stride * j0 - x_pos0 if j1 > j0 else t_old - x_pos0
    if lo < 0 or t_new - x_pos0 > x_win.shape[0] or t_old - x_pos0 < 0:
        raise ValueError("the token window does not hold the tokens the new rows need")
    seg = slice(stride * j0 - x_pos0, t_new - x_pos0)
    if j1 > j0:
        ent = compress(x_win[seg], g_win[seg], width, stride, rope_dim, theta,
                       pos_offset + stride * j0)
    else:
        ent = np.zeros((0, x_win.shape[1]), dtype=np.float64)
    raw = rotate_raw(x_win[t_old - x_pos0:t_new - x_pos0], t_old, rope_dim, theta)
    return j0, ent, raw


# --------------------------------------------------------------------------
# KV cache quantized after RoPE ("DeepSeek-V4.1-Flash vs Inkling", "Partial
# RoPE" row: the KV cache is quantized after RoPE; the pages give no
# format).  Read here as 8-bit floats E4M3 of the OCP 8-bit floating point
# specification (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
# no infinities, S.1111.111 the only NaN, largest finite 448) with one fp32
# scale per cache row: scale = max|row| / 448 (1 for an all-zero row), code
# = the E4M3 value nearest to x / scale, ties to the even code, magnitudes
# above 448 saturated.  The division and the scale are taken in fp32, the
# precision the codes are decided in on the GPU.
# --------------------------------------------------------------------------
def e4m3_values() -> np.ndarray:
    """The value of each of the 256 E4M3 codes (NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 0xF, c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = sign * 2.0 ** -6 * (m / 8.0)           # subnormal
        else:
            vals[c] = sign * 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return vals


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """Round each (finite) value to the nearest E4M3 code, ties to the even
    code, saturating at +-448; the sign of zero is kept."""
    y = np.asarray(y, dtype=np.float64)
    pos = e4m3_values()[:127]               # codes 0..126: 0, subnormals, normals to 448
    a = np.minimum(np.abs(y), pos[-1])
    hi = np.clip(np.searchsorted(pos, a, side="left"), 0, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - pos[lo], pos[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(y), code | np.uint8(0x80), code).astype(np.uint8)


def quantize_fp8_rows(rows: np.ndarray):
    """Cache rows [n, d] (the rotated values) -> (codes uint8 [n, d], scales
    fp32 [n]) with one scale per row."""
    r = np.asarray(rows, dtype=np.float32)
    amax = np.abs(r).max(axis=-1) if r.shape[-1] else np.zeros(r.shape[:-1], np.float32)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    y = r / scale[..., None]                  # fp32 division, as the codes are decided
    return e4m3_encode(y), scale


def dequantize_fp8_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """The cache rows the codes stand for: value(code) * scale, in fp64."""
    return e4m3_values()[np.asarray(codes)] * np.asarray(scales, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------
# Step 2: lightning indexer ("64 heads x 128 dims, ReLU scores weighted per
# head") and top-k ("keeps the top 1,024 entries")
# --------------------------------------------------------------------------
def index_scores(q_idx: np.ndarray, w: np.ndarray, k_idx: np.ndarray) -> np.ndarray:
    """s[t, j] = sum_h w[t, h] * ReLU(q_idx[t, h, :] . k_idx[j, :]).

    q_idx [Tq, H_I, d_I], w [Tq, H_I], k_idx [N, d_I] -> s [Tq, N]."""
    q_idx = np.asarray(q_idx, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k_idx = np.asarray(k_idx, dtype=np.float64)
    dots = np.matmul(q_idx, k_idx.T)                      # [Tq, H_I, N]
    return np.matmul(w[:, None, :], np.maximum(dots, 0.0))[:, 0, :]


def topk_select(scores: np.ndarray, n_vis: int, k: int) -> np.ndarray:
    """Indices of the k largest scores among entries 0..n_vis-1.

    Ties go to the lower index (a stable sort on (-score, index)); the kept
    indices are returned in ascending order, padded with -1 to length k."""
    out = np.full((k,), -1, dtype=np.int64)
    if n_vis <= 0:
        return out
    s = np.asarray(scores[:n_vis], dtype=np.float64)
    j = np.arange(n_vis, dtype=np.int64)
    order = np.lexsort((j, -s))  # primary key -score, then index
    keep = np.sort(order[:min(k, n_vis)])
    out[:keep.size] = keep
    return out


def index_topk(q_idx, w, k_idx, q_pos, n_cmp: int, width: int, stride: int,
               k: int, rows=None) -> np.ndarray:
    """Indexer + top-k for one sequence.  q_idx [Tq, H_I, d_I], w [Tq, H_I],
    k_idx [N, d_I], q_pos [Tq].  `rows` restricts to a sample of query rows.
    Returns idx [len(rows), k]."""
    rows = np.arange(len(q_pos)) if rows is None else np.asarray(rows)
    out = np.full((len(rows), k), -1, dtype=np.int64)
    for r0 in range(0, len(rows), 64):
        rr = rows[r0:r0 + 64]
        s = index_scores(np.asarray(q_idx)[rr], np.asarray(w)[rr], k_idx)
        for i, r in enumerate(rr):
            nv = n_visible(int(q_pos[r]), n_cmp, width, stride)
            out[r0 + i] = topk_select(s[i], nv, k)
    return out


# --------------------------------------------------------------------------
# Steps 3 and 4: shared-KV MQA over the gathered entries + window, with the
# sink in the denominator and the inverse output rotation
# --------------------------------------------------------------------------
def attend(q: np.ndarray, t: int, rows: np.ndarray, sink: np.ndarray, scale: float,
           rope_dim: int, theta) -> np.ndarray:
    """One query token.  q [H, d] (unrotated), rows [R, d] (rotated entries,
    each both key and value), sink [H].

    a_i = exp(z_i) / (exp(sink_h) + sum_i exp(z_i)), z_i = scale * (R(t) q_h) . r_i
    o_h = sum_i a_i r_i, then the trailing rope dims of o_h rotated at -t.
    Under YaRN the scale carries the attention temperature."""
    scale = scale * attention_temperature(theta)
    qh = rope(q, t, rope_dim, theta)
    sink = np.asarray(sink, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    H, d = qh.shape
    if rows.shape[0] == 0:
        return np.zeros((H, d), dtype=np.float64)
    z = (qh @ rows.T) * scale
    m = np.maximum(z.max(axis=1), sink)
    e = np.exp(z - m[:, None])
    den = np.exp(sink - m) + e.sum(axis=1)
    o = (e @ rows) / den[:, None]
    return rope(o, -t, rope_dim, theta)


def gather_rows(kv_cmp_b: np.ndarray, sel: np.ndarray, kv_raw_b: np.ndarray, t: int,
                window: int, raw_pos0: int, n_raw: int) -> np.ndarray:
    """The selected compressed entries followed by the window's raw rows."""
    sel = np.asarray(sel, dtype=np.int64)
    sel = sel[sel >= 0]
    win = window_tokens(t, window, raw_pos0, n_raw)
    parts = [np.asarray(kv_cmp_b)[sel].astype(np.float64),
             np.asarray(kv_raw_b)[win - raw_pos0].astype(np.float64)]
    return np.concatenate(parts, axis=0)


def sparse_attn(q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink, scale, window,
                rope_dim, theta, rows=None) -> np.ndarray:
    """CSA attention for one sequence: q [Tq, H, d], q_pos [Tq], kv_cmp [N, d],
    idx [Tq, k], kv_raw [R, d].  Returns out [len(rows), H, d]."""
    rows = np.arange(len(q_pos)) if rows is None else np.asarray(rows)
    out = []
    for r in rows:
        t = int(q_pos[r])
        kv = gather_rows(kv_cmp, idx[r], kv_raw, t, window, raw_pos0, n_raw)
        out.append(attend(np.asarray(q[r], dtype=np.float64), t, kv, sink, scale,
                          rope_dim, theta))
    return np.stack(out) if out else np.zeros((0,) + np.shape(q)[1:])


def hca_attn(q, q_pos, kv_cmp, n_cmp, kv_raw, raw_pos0, n_raw, sink, scale, window,
             width, stride, rope_dim, theta, rows=None) -> np.ndarray:
    """HCA attention for one sequence: every visible entry plus the window."""
    rows = np.arange(len(q_pos)) if rows is None else np.asarray(rows)
    out = []
    for r in rows:
        t = int(q_pos[r])
        sel = np.arange(n_visible(t, n_cmp, width, stride), dtype=np.int64)
        kv = gather_rows(kv_cmp, sel, kv_raw, t, window, raw_pos0, n_raw)
        out.append(attend(np.asarray(q[r], dtype=np.float64), t, kv, sink, scale,
                          rope_dim, theta))
    return np.stack(out) if out else np.zeros((0,) + np.shape(q)[1:])


# --------------------------------------------------------------------------
# The whole layer on one prefill sequence (compress -> index -> top-k ->
# attend), as the "Compressed Sparse Attention" row orders the steps.
# --------------------------------------------------------------------------
def csa_prefill_layer(x, g, q_idx, w, k_idx, q, sink, *, width, stride, topk, window,
                      rope_dim, theta, scale, pos_offset=0, rows=None):
    """Returns (kv_cmp, kv_raw, idx[rows], out[rows]) for one sequence whose
    tokens sit at positions 0..T-1 and are all queries."""
    T = np.shape(x)[0]
    kv_cmp = compress(x, g, width, stride, rope_dim, theta, pos_offset)
    kv_raw = rotate_raw(x, 0, rope_dim, theta)
    q_pos = np.arange(T)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    idx = index_topk(q_idx, w, k_idx, q_pos, kv_cmp.shape[0], width, stride, topk, rows)
    full_idx = np.full((T, topk), -1, dtype=np.int64)
    full_idx[rows] = idx
    out = sparse_attn(q, q_pos, kv_cmp, full_idx, kv_raw, 0, T, sink, scale, window,
                      rope_dim, theta, rows)
    return kv_cmp, kv_raw, idx, out


# --------------------------------------------------------------------------
# HCA on one prefill sequence ("Heavily Compressed Attention" row: every 128
# tokens pooled into one entry, dense shared-KV attention over all of them
# plus a 128-token window), every token a causal query
# --------------------------------------------------------------------------
def hca_prefill_layer(x, g, q, sink, *, window, rope_dim, theta, scale, width=128, stride=128,
                      pos_offset=0, rows=None):
    """Returns (kv_cmp, kv_raw, out[rows]) for one sequence whose tokens sit
    at positions 0..T-1: compression, then each query attends to every entry
    visible to it and its window."""
    T = np.shape(x)[0]
    kv_cmp = compress(x, g, width, stride, rope_dim, theta, pos_offset)
    kv_raw = rotate_raw(x, 0, rope_dim, theta)
    out = hca_attn(q, np.arange(T), kv_cmp, kv_cmp.shape[0], kv_raw, 0, T, sink, scale, window,
                   width, stride, rope_dim, theta, rows)
    return kv_cmp, kv_raw, out
