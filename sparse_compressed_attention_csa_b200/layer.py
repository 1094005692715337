"""User-level entry points: allocate outputs and workspace with torch, then
call the C ABI.  Every step runs in the CUDA library.

    decode: csa_decode(p, q, q_idx, w, k_idx, kv_cmp, kv_raw, ...) -> (idx, out)
    prefill: csa_prefill(p, x, gate, q_idx, w, k_idx, q, sink) -> (kv_cmp, kv_raw, idx, out)
    HCA decode: hca_decode(p, q, kv_cmp, kv_raw, ...) -> out
    HCA prefill: hca_prefill(p, x, gate, q, sink) -> (kv_cmp, kv_raw, out)
    CSA2 reuse layer: reuse_attn(p, q, ..., kv_cmp, idx, ...) -> out
    decode-time append: append_tokens(p, x, gate, x_pos0, t_old, t_new, ...)
    FP8 caches: quantize_fp8(rows) -> (codes, scales); csa_decode_fp8(...)
"""
from __future__ import annotations

import torch

from . import _lib as L


class Workspace:
    """A reusable device scratch buffer that grows on demand."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device or "cuda")
        return self.buf


def csa_decode(p: L.Params, q, q_pos, q_idx, w, k_idx, n_cmp, kv_cmp, kv_raw, raw_pos0, n_raw,
               sink, ws: Workspace | None = None, idx=None, out=None, stream=None):
    """Indexer + top-k + sparse attention for Tq query tokens per sequence."""
    ws = ws or Workspace(q.device)
    B, Tq = q_pos.shape
    n_max = k_idx.shape[1]
    if idx is None:
        idx = torch.empty((B, Tq, p.topk), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    nb = L.csa_workspace_size(p, L.CSA_OP_INDEX_TOPK, B, Tq, n_max)
    L.csa_index_topk(p, q_idx, w, k_idx, q_pos, n_cmp, idx, ws.get(nb), stream)
    nb = L.csa_workspace_size(p, L.CSA_OP_SPARSE_ATTN, B, Tq, kv_cmp.shape[1])
    L.csa_sparse_attn(p, q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink, out, ws.get(nb),
                      stream)
    return idx, out


def csa_prefill(p: L.Params, x, gate, q_idx, w, k_idx, q, sink, ws: Workspace | None = None,
                stream=None):
    """The whole layer on B sequences of T tokens, every token a causal query."""
    ws = ws or Workspace(x.device)
    B, T, d = x.shape
    N = 0 if T < p.width else (T - p.width) // p.stride + 1
    dev = x.device
    kv_cmp = torch.empty((B, N, d), dtype=x.dtype, device=dev)
    kv_raw = torch.empty((B, T, d), dtype=x.dtype, device=dev)
    L.csa_compress(p, x, gate, kv_cmp, kv_raw, stream)
    q_pos = torch.arange(T, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    n_cmp = torch.full((B,), N, dtype=torch.int32, device=dev)
    raw_pos0 = torch.zeros((B,), dtype=torch.int32, device=dev)
    n_raw = torch.full((B,), T, dtype=torch.int32, device=dev)
    idx, out = csa_decode(p, q, q_pos, q_idx, w, k_idx, n_cmp, kv_cmp, kv_raw, raw_pos0, n_raw,
                          sink, ws, stream=stream)
    return kv_cmp, kv_raw, idx, out


def hca_decode(p: L.Params, q, q_pos, kv_cmp, n_cmp, kv_raw, raw_pos0, n_raw, sink,
               ws: Workspace | None = None, out=None, stream=None):
    ws = ws or Workspace(q.device)
    B, Tq = q_pos.shape
    if out is None:
        out = torch.empty_like(q)
    nb = L.csa_workspace_size(p, L.CSA_OP_HCA_ATTN, B, Tq, kv_cmp.shape[1])
    L.hca_attn(p, q, q_pos, kv_cmp, n_cmp, kv_raw, raw_pos0, n_raw, sink, out, ws.get(nb), stream)
    return out


def reuse_attn(p: L.Params, q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink,
               ws: Workspace | None = None, out=None, stream=None):
    """Reuse layers of CSA2 ("CSA2 encoder layers (2x compression, Full +
    Reuse)": the rest reuse that KV and its top-512 selection): each layer's
    queries q [R][B][Tq][H][d] and sink [R][H] over the entries and indices a
    Full layer produced, all R layers in one call (a single layer:
    q [B][Tq][H][d], sink [H])."""
    ws = ws or Workspace(q.device)
    single = q.dim() == 4
    if single:
        q, sink = q.unsqueeze(0), sink.unsqueeze(0)
    if out is None:
        out = torch.empty_like(q)
    elif single:
        out = out.unsqueeze(0)
    R = q.shape[0]
    B, Tq = q_pos.shape
    nb = L.csa_workspace_size(p, L.CSA_OP_SPARSE_ATTN, R * B, Tq, kv_cmp.shape[1])
    L.csa_reuse_attn(p, q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink, out, ws.get(nb),
                     stream)
    return out[0] if single else out


def hca_prefill(p: L.Params, x, gate, q, sink, ws: Workspace | None = None, out=None,
                stream=None):
    """HCA on B sequences of T tokens, every token a causal query ("Heavily
    Compressed Attention" row: every 128 tokens pooled into one entry, dense
    attention over all of them plus a 128-token window); p.width and
    p.stride give the pooling."""
    ws = ws or Workspace(x.device)
    B, T, d = x.shape
    N = 0 if T < p.width else (T - p.width) // p.stride + 1
    dev = x.device
    kv_cmp = torch.empty((B, N, d), dtype=x.dtype, device=dev)
    kv_raw = torch.empty((B, T, d), dtype=x.dtype, device=dev)
    L.csa_compress(p, x, gate, kv_cmp, kv_raw, stream)
    q_pos = torch.arange(T, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    n_cmp = torch.full((B,), N, dtype=torch.int32, device=dev)
    raw_pos0 = torch.zeros((B,), dtype=torch.int32, device=dev)
    out = hca_decode(p, q, q_pos, kv_cmp, n_cmp, kv_raw, raw_pos0, n_cmp.new_full((B,), T), sink,
                     ws, out, stream)
    return kv_cmp, kv_raw, out


def append_tokens(p: L.Params, x, gate, x_pos0, t_old, t_new, max_new: int, kv_cmp,
                  kv_raw=None, raw_pos0=None, stream=None):
    """Decode-time compression: write the entries and rotated raw rows that
    tokens t_old[b] .. t_new[b] - 1 complete into the caches (entry j at
    row j of kv_cmp, token t at row t - raw_pos0[b] of kv_raw); x, gate hold
    token x_pos0[b] + i at row i."""
    L.csa_compress_append(p, x, gate, x_pos0, t_old, t_new, max_new, kv_cmp, kv_raw, raw_pos0,
                          stream)


def quantize_fp8(rows, stream=None):
    """Cache rows [..., d] (rotated) -> (E4M3 codes uint8 [..., d], fp32
    scales [...]), one scale per row: the KV cache quantized after RoPE."""
    codes = torch.empty(rows.shape, dtype=torch.uint8, device=rows.device)
    scales = torch.empty(rows.shape[:-1], dtype=torch.float32, device=rows.device)
    L.csa_quantize_fp8(rows, codes, scales, stream)
    return codes, scales


def csa_decode_fp8(p: L.Params, q, q_pos, q_idx, w, k_idx, n_cmp, kv_cmp, cmp_scale, kv_raw,
                   raw_scale, raw_pos0, n_raw, sink, ws: Workspace | None = None, idx=None,
                   out=None, stream=None):
    """csa_decode over FP8 caches (codes and row scales from quantize_fp8)."""
    ws = ws or Workspace(q.device)
    B, Tq = q_pos.shape
    n_max = k_idx.shape[1]
    if idx is None:
        idx = torch.empty((B, Tq, p.topk), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    nb = L.csa_workspace_size(p, L.CSA_OP_INDEX_TOPK, B, Tq, n_max)
    L.csa_index_topk(p, q_idx, w, k_idx, q_pos, n_cmp, idx, ws.get(nb), stream)
    nb = L.csa_workspace_size(p, L.CSA_OP_SPARSE_ATTN, B, Tq, kv_cmp.shape[1])
    L.csa_sparse_attn_fp8(p, q, q_pos, kv_cmp, cmp_scale, idx, kv_raw, raw_scale, raw_pos0, n_raw,
                          sink, out, ws.get(nb), stream)
    return idx, out
