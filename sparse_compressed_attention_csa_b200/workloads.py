"""Seeded synthetic inputs for the CSA / HCA attention layer.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no pooling, no RoPE, no scoring, no softmax).  The
CUDA path (through the C-ABI binding) and the fp64 oracle both receive the
arrays it returns, so they always see bit-identical inputs.

Shapes follow the layer as stated on "DeepSeek-V4-Pro vs Inkling"
(archdiff.com), component table, rows "Compressed Sparse Attention",
"Heavily Compressed Attention", "Partial RoPE" and "Output gate + sink",
and the raw config fields on "DeepSeek-V4-Pro" (llm-atlas) (`head_dim` 512,
`num_attention_heads` 128, `index_n_heads` 64, `index_head_dim` 128,
`index_topk` 1024, `sliding_window` 128, `qk_rope_head_dim` 64).

Recipe (one `numpy.random.Generator(PCG64)` stream per tensor, spawned from
`SeedSequence(seed)` in the fixed order x, g, k_idx, q_idx, w, q, sink,
kv_cmp, kv_raw):

* token KV `x` and gate logits `g`: N(0, 1);
* indexer keys / queries: integers uniform on [-R, R] (R = 8, or 3 for the
  tiny fp32 workload), so every indexer score is an exact fp32 value;
* indexer head weights: 2**e, e uniform on the workload's exponent set;
* queries `q`, sink logits, pre-compressed caches: N(0, 1);
* bf16 workloads round every fp32 draw to bf16 (round to nearest even) and
  hand out the raw 16-bit patterns as `uint16` arrays.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np

_STREAMS = ("x", "g", "k_idx", "q_idx", "w", "q", "sink", "kv_cmp", "kv_raw", "q_reuse",
            "sink_reuse")
_CHUNK = 1 << 24


@dataclass(frozen=True)
class Workload:
    """One synthetic workload of the layer.

    kind: "csa_decode" (pre-compressed caches, one query per sequence),
          "csa_prefill" (token KV + gates are pooled in the path, every
          token is a causal query), "hca_decode" or "hca_prefill".
    """

    name: str
    kind: str
    dtype: str  # "f32" or "bf16"
    B: int
    T: int
    seed: int
    d: int = 512
    rope_dim: int = 64
    theta: float = 10000.0
    n_heads: int = 128
    idx_heads: int = 64
    idx_dim: int = 128
    topk: int = 1024
    window: int = 128
    width: int = 8
    stride: int = 4
    pos_offset: int = 0
    int_range: int = 8
    w_exps: tuple = (-2, -1, 0, 1, 2)
    rope_factor: float = 1.0     # YaRN factor (1: plain RoPE)
    rope_orig_ctx: int = 0       # YaRN original context
    rope_beta_fast: float = 32.0
    rope_beta_slow: float = 1.0
    reuse_layers: int = 0        # layers attending over this layer's entries and selection
    kv_fp8: bool = False         # attention over the caches quantized to E4M3 after RoPE

    @property
    def scale(self) -> float:
        return float(1.0 / np.sqrt(self.d))

    @property
    def n_cmp(self) -> int:
        """Entries pooled from T tokens: floor((T - width) / stride) + 1."""
        if self.T < self.width:
            return 0
        return (self.T - self.width) // self.stride + 1

    @property
    def Tq(self) -> int:
        return self.T if self.kind in ("csa_prefill", "hca_prefill") else 1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the layer is measured and checked on.
TINY_F32 = Workload(
    name="tiny_csa_f32_T256", kind="csa_prefill", dtype="f32", B=1, T=256, seed=1,
    n_heads=4, idx_heads=4, idx_dim=32, topk=16, window=16, int_range=3,
    w_exps=(-1, 0, 1))
CSA_DECODE_64K = Workload(
    name="csa_decode_bs32_ctx65536", kind="csa_decode", dtype="bf16", B=32, T=65536, seed=2)
CSA_PREFILL_8K = Workload(
    name="csa_prefill_T8192", kind="csa_prefill", dtype="bf16", B=1, T=8192, seed=3)
CSA_DECODE_1M = Workload(
    name="csa_decode_bs4_ctx1048576", kind="csa_decode", dtype="bf16", B=4, T=1048576, seed=4)
HCA_DECODE_128K = Workload(
    name="hca_decode_bs16_ctx131072", kind="hca_decode", dtype="bf16", B=16, T=131072, seed=5,
    width=128, stride=128)

# The compressed layers' extended RoPE ("Partial RoPE" rows: theta 160,000
# with YaRN, factor 16 over 65,536 tokens) on a decode batch whose context
# (128K tokens) runs past the original 64K.
CSA_DECODE_YARN = Workload(
    name="csa_decode_yarn_bs32_ctx131072", kind="csa_decode", dtype="bf16", B=32, T=131072,
    seed=6, theta=160000.0, rope_factor=16.0, rope_orig_ctx=65536)

# CSA2 ("DeepSeek-V4.1-Flash vs Inkling", row "CSA2 encoder layers (2x
# compression, Full + Reuse)": KV pooled 2 -> 1 and computed in 3 of 18
# layers, the rest reuse that KV and its top-512 selection; "Partial RoPE"
# row: theta 160,000 with YaRN): one Full layer and the 5 Reuse layers that
# share its entries, on the 64K-context decode batch.
CSA2_DECODE = Workload(
    name="csa2_decode_bs32_ctx65536", kind="csa_decode", dtype="bf16", B=32, T=65536, seed=7,
    width=2, stride=2, topk=512, theta=160000.0, rope_factor=16.0, rope_orig_ctx=65536,
    reuse_layers=5)

# The 64K-context decode batch over the KV cache quantized after RoPE
# ("DeepSeek-V4.1-Flash vs Inkling", "Partial RoPE" row), here E4M3 codes
# with one fp32 scale per row: the same inputs, the caches quantized once
# when written (outside the step).
CSA_DECODE_FP8 = Workload(
    name="csa_decode_fp8kv_bs32_ctx65536", kind="csa_decode", dtype="bf16", B=32, T=65536,
    seed=2, kv_fp8=True)

# HCA on a prefill sequence ("Heavily Compressed Attention" row: 128 tokens
# -> 1 entry, dense attention over every entry plus the window), the CSA
# prefill's length: 64 entries, every token a causal query.
HCA_PREFILL_8K = Workload(
    name="hca_prefill_T8192", kind="hca_prefill", dtype="bf16", B=1, T=8192, seed=8,
    width=128, stride=128)

WORKLOADS = {w.name: w for w in (TINY_F32, CSA_DECODE_64K, CSA_PREFILL_8K, CSA_DECODE_1M,
                                 HCA_DECODE_128K, CSA_DECODE_YARN, CSA2_DECODE,
                                 HCA_PREFILL_8K, CSA_DECODE_FP8)}


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the fp32 values they encode (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_f64(a: np.ndarray) -> np.ndarray:
    """Any generated array (fp32 values or bf16 bit patterns) as float64."""
    if a.dtype == np.uint16:
        return bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


class _Streams:
    def __init__(self, seed: int):
        kids = np.random.SeedSequence(seed).spawn(len(_STREAMS))
        self._g = {n: np.random.Generator(np.random.PCG64(s)) for n, s in zip(_STREAMS, kids)}

    def __getitem__(self, name: str) -> np.random.Generator:
        return self._g[name]


def _normal(rng: np.random.Generator, shape, bf16: bool) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if bf16 else np.float32)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        v = rng.standard_normal(e - s, dtype=np.float32)
        out[s:e] = bf16_bits(v) if bf16 else v
    return out.reshape(shape)


def _ints(rng: np.random.Generator, shape, r: int, bf16: bool) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if bf16 else np.float32)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        v = rng.integers(-r, r + 1, size=e - s).astype(np.float32)
        out[s:e] = bf16_bits(v) if bf16 else v
    return out.reshape(shape)


def generate(wl: Workload, keys=None) -> dict:
    """Draw every input of `wl` (or only those named in `keys`: each tensor
    has its own stream, so skipping one changes no other).

    Returned keys (shapes; bf16 workloads give uint16 bit patterns for the
    big tensors, fp32 elsewhere):

    * all kinds: q [B,Tq,H,d], sink [H] fp32, q_pos [B,Tq] int32
    * csa kinds: q_idx [B,Tq,H_I,d_I], w [B,Tq,H_I] fp32, k_idx [B,N,d_I],
      n_cmp [B] int32
    * prefill: x, g [B,T,d] (the caches are produced by pooling in the path)
    * decode kinds: kv_cmp [B,N,d], kv_raw [B,W,d] (already rotated caches),
      raw_pos0 [B], n_raw [B] int32
    * with reuse layers: q_reuse [R,B,Tq,H,d], sink_reuse [R,H] fp32
    """
    bf16 = wl.dtype == "bf16"
    st = _Streams(wl.seed)
    B, T, d, N, Tq = wl.B, wl.T, wl.d, wl.n_cmp, wl.Tq
    out: dict = {}
    want = (lambda k: True) if keys is None else (lambda k: k in keys)

    def normal(rng, shape, key):  # drawn only when wanted
        return _normal(rng, shape, bf16) if want(key) else None

    def ints(rng, shape, key):
        return _ints(rng, shape, wl.int_range, bf16) if want(key) else None

    prefill = wl.kind in ("csa_prefill", "hca_prefill")
    if prefill:
        out["x"] = normal(st["x"], (B, T, d), "x")
        out["g"] = normal(st["g"], (B, T, d), "g")
    if wl.kind in ("csa_prefill", "csa_decode"):
        out["k_idx"] = ints(st["k_idx"], (B, N, wl.idx_dim), "k_idx")
        out["q_idx"] = ints(st["q_idx"], (B, Tq, wl.idx_heads, wl.idx_dim), "q_idx")
        e = st["w"].integers(0, len(wl.w_exps), size=(B, Tq, wl.idx_heads))
        out["w"] = np.exp2(np.asarray(wl.w_exps, dtype=np.float32)[e]).astype(np.float32)
        out["n_cmp"] = np.full((B,), N, dtype=np.int32)
    out["q"] = normal(st["q"], (B, Tq, wl.n_heads, d), "q")
    out["sink"] = st["sink"].standard_normal(wl.n_heads, dtype=np.float32)
    if wl.reuse_layers > 0:
        R = wl.reuse_layers
        out["q_reuse"] = normal(st["q_reuse"], (R, B, Tq, wl.n_heads, d), "q_reuse")
        out["sink_reuse"] = st["sink_reuse"].standard_normal((R, wl.n_heads), dtype=np.float32)
    if prefill:
        out["q_pos"] = np.tile(np.arange(T, dtype=np.int32), (B, 1))
        out["raw_pos0"] = np.zeros((B,), dtype=np.int32)
        out["n_raw"] = np.full((B,), T, dtype=np.int32)
    else:
        out["q_pos"] = np.full((B, 1), T - 1, dtype=np.int32)
        out["kv_cmp"] = normal(st["kv_cmp"], (B, N, d), "kv_cmp")
        W = wl.window
        out["kv_raw"] = normal(st["kv_raw"], (B, W, d), "kv_raw")
        out["raw_pos0"] = np.full((B,), T - W, dtype=np.int32)
        out["n_raw"] = np.full((B,), W, dtype=np.int32)
        if wl.kind == "hca_decode":
            out["n_cmp"] = np.full((B,), N, dtype=np.int32)
    return {k: v for k, v in out.items() if v is not None}
