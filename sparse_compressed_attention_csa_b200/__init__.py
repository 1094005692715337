"""B200-native (sm_100a) Compressed Sparse Attention (CSA) and Heavily
Compressed Attention (HCA), DeepSeek-V4 style.

The four steps of the layer run as hand-written CUDA kernels behind the C ABI
in include/csa.h (libcsa.so); this package is its thin Python binding, with
the same names.  torch supplies device memory and streams.

    from sparse_compressed_attention_csa_b200 import Params, csa_index_topk, ...
"""
from ._lib import (  # noqa: F401
    CSA_BF16, CSA_F32, CSA_OP_COMPRESS, CSA_OP_HCA_ATTN, CSA_OP_INDEX_TOPK, CSA_OP_SPARSE_ATTN,
    CSA_OP_TOPK_SELECT, CsaError, Params, csa_compress, csa_compress_append, csa_index_scores,
    csa_index_topk,
    csa_index_topk_noalloc, csa_last_device_error_site, csa_launch_count, csa_poll_device_error,
    csa_quantize_fp8, csa_reuse_attn, csa_set_wait_limit_ns, csa_sparse_attn, csa_sparse_attn_fp8, csa_topk_select,
    csa_workspace_size, hca_attn, hca_attn_fp8, lib)

__all__ = [
    "Params", "CsaError", "csa_compress", "csa_compress_append", "csa_index_scores", "csa_topk_select",
    "csa_index_topk", "csa_index_topk_noalloc", "csa_sparse_attn", "hca_attn", "csa_workspace_size",
    "csa_poll_device_error", "csa_last_device_error_site", "csa_set_wait_limit_ns",
    "csa_launch_count", "csa_quantize_fp8", "csa_reuse_attn", "csa_sparse_attn_fp8", "hca_attn_fp8", "lib",
]
