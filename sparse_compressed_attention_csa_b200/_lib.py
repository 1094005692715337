"""ctypes binding of libcsa.so (the C ABI in include/csa.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Functions take torch CUDA tensors (torch is used for device
memory and streams), check dtype / contiguity / device, and pass raw
pointers and sizes through.  A missing library raises immediately: there is
no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_F32, CSA_BF16 = 0, 1
CSA_OP_COMPRESS, CSA_OP_INDEX_TOPK, CSA_OP_SPARSE_ATTN, CSA_OP_HCA_ATTN, CSA_OP_TOPK_SELECT = range(5)

STATUS = {
    0: "CSA_OK", 1: "CSA_ERR_INVALID_ARGUMENT", 2: "CSA_ERR_MISALIGNED",
    3: "CSA_ERR_UNSUPPORTED_SHAPE", 4: "CSA_ERR_UNSUPPORTED_DEVICE",
    5: "CSA_ERR_WORKSPACE_TOO_SMALL", 6: "CSA_ERR_CUDA", 7: "CSA_ERR_DEVICE_TIMEOUT",
    8: "CSA_ERR_DEVICE_BOUNDS",
}


class CsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class csa_params_t(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("rope_dim", ctypes.c_int32), ("theta", ctypes.c_float),
                ("scale", ctypes.c_float), ("n_heads", ctypes.c_int32),
                ("idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("window", ctypes.c_int32), ("width", ctypes.c_int32),
                ("stride", ctypes.c_int32), ("pos_offset", ctypes.c_int32),
                ("rope_factor", ctypes.c_float), ("rope_orig_ctx", ctypes.c_int32),
                ("rope_beta_fast", ctypes.c_float), ("rope_beta_slow", ctypes.c_float)]


@dataclass(frozen=True)
class Params:
    """Layer constants (defaults: the measured model's CSA layer)."""
    d: int = 512
    rope_dim: int = 64
    theta: float = 10000.0
    scale: float | None = None  # None -> 1/sqrt(d)
    n_heads: int = 128
    idx_heads: int = 64
    idx_dim: int = 128
    topk: int = 1024
    window: int = 128
    width: int = 8
    stride: int = 4
    pos_offset: int = 0
    rope_factor: float = 1.0      # YaRN factor s (1: plain RoPE)
    rope_orig_ctx: int = 0        # YaRN original context L
    rope_beta_fast: float = 32.0  # YaRN beta
    rope_beta_slow: float = 1.0   # YaRN alpha

    def c(self) -> csa_params_t:
        """The C struct, built once per (immutable) parameter set; the
        library only reads it during a call."""
        cs = self.__dict__.get("_c")
        if cs is None:
            sc = self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)
            cs = csa_params_t(self.d, self.rope_dim, self.theta, sc, self.n_heads,
                              self.idx_heads, self.idx_dim, self.topk, self.window, self.width,
                              self.stride, self.pos_offset, self.rope_factor, self.rope_orig_ctx,
                              self.rope_beta_fast, self.rope_beta_slow)
            object.__setattr__(self, "_c", cs)
        return cs


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_PP = ctypes.POINTER(csa_params_t)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library {LIB_PATH} is not built; run "
                          "sparse_compressed_attention_csa_b200.build.build() (there is no "
                          "CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.csa_abi_version.restype = ctypes.c_int
    lib.csa_status_string.restype = ctypes.c_char_p
    lib.csa_status_string.argtypes = [ctypes.c_int]
    lib.csa_last_error_detail.restype = ctypes.c_char_p
    lib.csa_workspace_size.argtypes = [_PP, ctypes.c_int, _I, _I, _I,
                                       ctypes.POINTER(ctypes.c_size_t)]
    lib.csa_compress.argtypes = [_PP, ctypes.c_int, _P, _P, _I, _I, _P, _P, _P]
    lib.csa_compress_append.argtypes = [_PP, ctypes.c_int, _P, _P, _P, _I, _I, _P, _P, _I, _P, _I,
                                        _P, _P, _I, _P]
    lib.csa_index_scores.argtypes = [_PP, ctypes.c_int, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]
    lib.csa_topk_select.argtypes = [_PP, _P, _P, _P, _I, _I, _I, _P, _P, ctypes.c_size_t, _P]
    lib.csa_index_topk.argtypes = [_PP, ctypes.c_int, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P,
                                   ctypes.c_size_t, _P]
    lib.csa_sparse_attn.argtypes = [_PP, ctypes.c_int, _P, _P, _P, _P, _I, _P, _P, _P, _I, _P,
                                    _I, _I, _P, _P, ctypes.c_size_t, _P]
    lib.hca_attn.argtypes = list(lib.csa_sparse_attn.argtypes)
    lib.csa_reuse_attn.argtypes = [_PP, ctypes.c_int, _I] + list(lib.csa_sparse_attn.argtypes[2:])
    lib.csa_quantize_fp8.argtypes = [ctypes.c_int, _P, ctypes.c_int64, _I, _P, _P, _P]
    lib.csa_sparse_attn_fp8.argtypes = [_PP, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I, _P, _I,
                                        _I, _P, _P, ctypes.c_size_t, _P]
    lib.hca_attn_fp8.argtypes = list(lib.csa_sparse_attn_fp8.argtypes)
    lib.csa_index_topk_noalloc.argtypes = [_PP, ctypes.c_int, _P, _P, _P, _P, _P, _I, _I, _I, _P,
                                           _P]
    lib.csa_poll_device_error.argtypes = [_P]
    lib.csa_launch_count.restype = ctypes.c_uint64
    lib.csa_launch_count.argtypes = []
    lib.csa_set_wait_limit_ns.restype = None
    lib.csa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.csa_last_device_error_site.restype = ctypes.c_int32
    lib.csa_last_device_error_site.argtypes = []
    for f in ("csa_workspace_size", "csa_compress", "csa_index_scores", "csa_topk_select",
              "csa_index_topk", "csa_sparse_attn", "hca_attn", "csa_poll_device_error",
              "csa_compress_append", "csa_quantize_fp8", "csa_sparse_attn_fp8", "hca_attn_fp8",
              "csa_reuse_attn",
              "csa_index_topk_noalloc"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def lib():
    return _load()


def _check(st: int):
    if st != 0:
        raise CsaError(st, _load().csa_last_error_detail().decode(errors="replace"))


def _ptr(t):
    # a plain int: the c_void_p argtypes convert it
    return None if t is None else t.data_ptr()


def _stream(stream):
    """The cudaStream_t of `stream`, or of the current stream of the current
    device (read through torch's raw-stream query, which skips building a
    Stream object on every call)."""
    import torch
    if stream is not None:
        return stream.cuda_stream
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return raw(torch._C._cuda_getDevice())
    return torch.cuda.current_stream().cuda_stream


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype == torch.float32:
        return CSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _req(t, name, dtype=None, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t


_ws_sizes = {}


def csa_workspace_size(p: Params, op: int, B: int, Tq: int, n_max: int) -> int:
    """Bytes of workspace the call `op` needs (a pure function of the
    arguments and the current device, so answers are kept per device)."""
    import torch
    key = (p, op, B, Tq, n_max, torch.cuda.current_device() if torch.cuda.is_available() else -1)
    nb = _ws_sizes.get(key)
    if nb is None:
        n = ctypes.c_size_t(0)
        _check(_load().csa_workspace_size(ctypes.byref(p.c()), op, B, Tq, n_max,
                                          ctypes.byref(n)))
        nb = _ws_sizes[key] = int(n.value)
    return nb


def csa_compress(p: Params, x, gate, kv_cmp_out, kv_raw_rot_out=None, stream=None):
    """x, gate [B][T][d] -> kv_cmp_out [B][N][d] (+ kv_raw_rot_out [B][T][d])."""
    _req(x, "x", ndim=3)
    _req(gate, "gate", x.dtype, 3)
    _req(kv_cmp_out, "kv_cmp_out", x.dtype, 3)
    if kv_raw_rot_out is not None:
        _req(kv_raw_rot_out, "kv_raw_rot_out", x.dtype, 3)
    B, T, d = x.shape
    _check(_load().csa_compress(ctypes.byref(p.c()), _dtype_code(x), _ptr(x), _ptr(gate), B, T,
                                _ptr(kv_cmp_out), _ptr(kv_raw_rot_out), _stream(stream)))


def csa_compress_append(p: Params, x, gate, x_pos0, t_old, t_new, max_new: int, kv_cmp,
                        kv_raw=None, raw_pos0=None, stream=None):
    """Entries and raw rows completed by tokens t_old[b] .. t_new[b] - 1:
    x, gate [B][L][d] (row i = token x_pos0[b] + i) -> rows of kv_cmp
    [B][n_cap][d] (entry j at row j) and kv_raw [B][raw_cap][d] (token t at
    row t - raw_pos0[b])."""
    import torch
    _req(x, "x", ndim=3)
    _req(gate, "gate", x.dtype, 3)
    for t, n in ((x_pos0, "x_pos0"), (t_old, "t_old"), (t_new, "t_new")):
        _req(t, n, torch.int32, 1)
    _req(kv_cmp, "kv_cmp", x.dtype, 3)
    if kv_raw is not None:
        _req(kv_raw, "kv_raw", x.dtype, 3)
        _req(raw_pos0, "raw_pos0", torch.int32, 1)
    B, L, d = x.shape
    _check(_load().csa_compress_append(
        ctypes.byref(p.c()), _dtype_code(x), _ptr(x), _ptr(gate), _ptr(x_pos0), B, L, _ptr(t_old),
        _ptr(t_new), int(max_new), _ptr(kv_cmp), kv_cmp.shape[1], _ptr(kv_raw),
        _ptr(raw_pos0), kv_raw.shape[1] if kv_raw is not None else 0, _stream(stream)))


def csa_index_scores(p: Params, q_idx, w, k_idx, q_pos, n_cmp, scores, stream=None):
    """q_idx [B][Tq][H_I][d_I], w [B][Tq][H_I], k_idx [B][n_max][d_I] -> scores [B][Tq][n_max]."""
    import torch
    _req(q_idx, "q_idx", ndim=4)
    _req(w, "w", torch.float32, 3)
    _req(k_idx, "k_idx", q_idx.dtype, 3)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(n_cmp, "n_cmp", torch.int32, 1)
    _req(scores, "scores", torch.float32, 3)
    B, Tq = q_pos.shape
    n_max = k_idx.shape[1]
    _check(_load().csa_index_scores(ctypes.byref(p.c()), _dtype_code(q_idx), _ptr(q_idx), _ptr(w),
                                    _ptr(k_idx), _ptr(q_pos), _ptr(n_cmp), B, Tq, n_max,
                                    _ptr(scores), _stream(stream)))


def csa_topk_select(p: Params, scores, q_pos, n_cmp, idx_out, ws=None, stream=None):
    """scores [B][Tq][n_max] fp32 -> idx_out [B][Tq][topk] int32."""
    import torch
    _req(scores, "scores", torch.float32, 3)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(n_cmp, "n_cmp", torch.int32, 1)
    _req(idx_out, "idx_out", torch.int32, 3)
    B, Tq, n_max = scores.shape
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().csa_topk_select(ctypes.byref(p.c()), _ptr(scores), _ptr(q_pos), _ptr(n_cmp),
                                   B, Tq, n_max, _ptr(idx_out), _ptr(ws), nb, _stream(stream)))


def csa_index_topk(p: Params, q_idx, w, k_idx, q_pos, n_cmp, idx_out, ws, stream=None):
    """Indexer + top-k; ws: csa_workspace_size(CSA_OP_INDEX_TOPK) bytes."""
    import torch
    _req(q_idx, "q_idx", ndim=4)
    _req(w, "w", torch.float32, 3)
    _req(k_idx, "k_idx", q_idx.dtype, 3)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(n_cmp, "n_cmp", torch.int32, 1)
    _req(idx_out, "idx_out", torch.int32, 3)
    B, Tq = q_pos.shape
    n_max = k_idx.shape[1]
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().csa_index_topk(ctypes.byref(p.c()), _dtype_code(q_idx), _ptr(q_idx), _ptr(w),
                                  _ptr(k_idx), _ptr(q_pos), _ptr(n_cmp), B, Tq, n_max,
                                  _ptr(idx_out), _ptr(ws), nb, _stream(stream)))


def csa_index_topk_noalloc(p: Params, q_idx, w, k_idx, q_pos, n_cmp, idx_out, stream=None):
    """Indexer + top-k without a workspace, for callers that cannot allocate
    device memory.  Scores go to an 8 MiB array built into the library
    (B * Tq * n_max <= 2**21); calls that overlap on the GPU share it and race."""
    import torch
    _req(q_idx, "q_idx", ndim=4)
    _req(w, "w", torch.float32, 3)
    _req(k_idx, "k_idx", q_idx.dtype, 3)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(n_cmp, "n_cmp", torch.int32, 1)
    _req(idx_out, "idx_out", torch.int32, 3)
    B, Tq = q_pos.shape
    n_max = k_idx.shape[1]
    _check(_load().csa_index_topk_noalloc(ctypes.byref(p.c()), _dtype_code(q_idx), _ptr(q_idx),
                                          _ptr(w), _ptr(k_idx), _ptr(q_pos), _ptr(n_cmp), B, Tq,
                                          n_max, _ptr(idx_out), _stream(stream)))


def _attn(fn, p, q, q_pos, kv_cmp, sel, kv_raw, raw_pos0, n_raw, sink, out, ws, stream):
    import torch
    _req(q, "q", ndim=4)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(kv_cmp, "kv_cmp", q.dtype, 3)
    _req(kv_raw, "kv_raw", q.dtype, 3)
    _req(raw_pos0, "raw_pos0", torch.int32, 1)
    _req(n_raw, "n_raw", torch.int32, 1)
    _req(sink, "sink", torch.float32, 1)
    _req(out, "out", q.dtype, 4)
    B, Tq = q_pos.shape
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(fn(ctypes.byref(p.c()), _dtype_code(q), _ptr(q), _ptr(q_pos), _ptr(kv_cmp), _ptr(sel),
              kv_cmp.shape[1], _ptr(kv_raw), _ptr(raw_pos0), _ptr(n_raw), kv_raw.shape[1],
              _ptr(sink), B, Tq, _ptr(out), _ptr(ws), nb, _stream(stream)))


def csa_sparse_attn(p: Params, q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink, out,
                    ws=None, stream=None):
    """q [B][Tq][H][d], idx [B][Tq][topk] -> out [B][Tq][H][d]."""
    import torch
    _req(idx, "idx", torch.int32, 3)
    _attn(_load().csa_sparse_attn, p, q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink, out,
          ws, stream)


def csa_reuse_attn(p: Params, q, q_pos, kv_cmp, idx, kv_raw, raw_pos0, n_raw, sink, out, ws=None,
                   stream=None):
    """CSA2 Reuse layers: q [R][B][Tq][H][d], sink [R][H] -> out [R][B][Tq][H][d],
    every layer over the same entries, selection (idx [B][Tq][topk]) and window."""
    import torch
    _req(q, "q", ndim=5)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(kv_cmp, "kv_cmp", q.dtype, 3)
    _req(idx, "idx", torch.int32, 3)
    _req(kv_raw, "kv_raw", q.dtype, 3)
    _req(raw_pos0, "raw_pos0", torch.int32, 1)
    _req(n_raw, "n_raw", torch.int32, 1)
    _req(sink, "sink", torch.float32, 2)
    _req(out, "out", q.dtype, 5)
    R = q.shape[0]
    B, Tq = q_pos.shape
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_load().csa_reuse_attn(ctypes.byref(p.c()), _dtype_code(q), R, _ptr(q), _ptr(q_pos),
                                  _ptr(kv_cmp), _ptr(idx), kv_cmp.shape[1], _ptr(kv_raw),
                                  _ptr(raw_pos0), _ptr(n_raw), kv_raw.shape[1], _ptr(sink), B, Tq,
                                  _ptr(out), _ptr(ws), nb, _stream(stream)))


def hca_attn(p: Params, q, q_pos, kv_cmp, n_cmp, kv_raw, raw_pos0, n_raw, sink, out, ws=None,
             stream=None):
    """Dense attention over every visible entry + window."""
    import torch
    _req(n_cmp, "n_cmp", torch.int32, 1)
    _attn(_load().hca_attn, p, q, q_pos, kv_cmp, n_cmp, kv_raw, raw_pos0, n_raw, sink, out, ws,
          stream)


def csa_launch_count() -> int:
    """Kernels launched (or captured) by the library so far in this process."""
    return int(_load().csa_launch_count())


def csa_set_wait_limit_ns(ns: int = 0):
    """Limit of every bounded wait in the library's kernels (0: the 2 s
    default).  Read at launch; a diagnostic for exercising the timeout path."""
    _load().csa_set_wait_limit_ns(int(ns))


def csa_poll_device_error(stream=None):
    _check(_load().csa_poll_device_error(_stream(stream)))


def csa_last_device_error_site() -> int:
    """Kernel source line of the check behind the last device error polled."""
    return int(_load().csa_last_device_error_site())


def csa_quantize_fp8(rows, codes, scales, stream=None):
    """Cache rows [..., d] (bf16 or fp32, already rotated) -> E4M3 codes
    [..., d] uint8 and one fp32 scale per row [...]."""
    import torch
    _req(rows, "rows")
    _req(codes, "codes", torch.uint8, rows.dim())
    _req(scales, "scales", torch.float32, rows.dim() - 1)
    d = rows.shape[-1]
    n = rows.numel() // d if d else 0
    if tuple(codes.shape) != tuple(rows.shape) or tuple(scales.shape) != tuple(rows.shape[:-1]):
        raise ValueError("codes must match rows and scales its leading dims")
    _check(_load().csa_quantize_fp8(_dtype_code(rows), _ptr(rows), n, d, _ptr(codes), _ptr(scales),
                                    _stream(stream)))


def _attn_fp8(fn, p, q, q_pos, kv_cmp, cmp_scale, sel, kv_raw, raw_scale, raw_pos0, n_raw, sink,
              out, ws, stream):
    import torch
    _req(q, "q", torch.bfloat16, 4)
    _req(q_pos, "q_pos", torch.int32, 2)
    _req(kv_cmp, "kv_cmp", torch.uint8, 3)
    _req(cmp_scale, "cmp_scale", torch.float32, 2)
    _req(kv_raw, "kv_raw", torch.uint8, 3)
    _req(raw_scale, "raw_scale", torch.float32, 2)
    _req(raw_pos0, "raw_pos0", torch.int32, 1)
    _req(n_raw, "n_raw", torch.int32, 1)
    _req(sink, "sink", torch.float32, 1)
    _req(out, "out", torch.bfloat16, 4)
    B, Tq = q_pos.shape
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(fn(ctypes.byref(p.c()), _ptr(q), _ptr(q_pos), _ptr(kv_cmp), _ptr(cmp_scale), _ptr(sel),
              kv_cmp.shape[1], _ptr(kv_raw), _ptr(raw_scale), _ptr(raw_pos0), _ptr(n_raw),
              kv_raw.shape[1], _ptr(sink), B, Tq, _ptr(out), _ptr(ws), nb, _stream(stream)))


def csa_sparse_attn_fp8(p: Params, q, q_pos, kv_cmp, cmp_scale, idx, kv_raw, raw_scale, raw_pos0,
                        n_raw, sink, out, ws=None, stream=None):
    """As csa_sparse_attn over FP8 caches: kv_cmp [B][n_max][d] and kv_raw
    [B][raw_max][d] E4M3 codes with row scales [B][n_max], [B][raw_max]."""
    import torch
    _req(idx, "idx", torch.int32, 3)
    _attn_fp8(_load().csa_sparse_attn_fp8, p, q, q_pos, kv_cmp, cmp_scale, idx, kv_raw, raw_scale,
              raw_pos0, n_raw, sink, out, ws, stream)


def hca_attn_fp8(p: Params, q, q_pos, kv_cmp, cmp_scale, n_cmp, kv_raw, raw_scale, raw_pos0,
                 n_raw, sink, out, ws=None, stream=None):
    """As hca_attn over FP8 caches (codes and row scales)."""
    import torch
    _req(n_cmp, "n_cmp", torch.int32, 1)
    _attn_fp8(_load().hca_attn_fp8, p, q, q_pos, kv_cmp, cmp_scale, n_cmp, kv_raw, raw_scale,
              raw_pos0, n_raw, sink, out, ws, stream)
