"""fp64 CPU oracle of the CSA / HCA attention layer (test infrastructure only).

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline legs
may import this package.  It shares no code with the CUDA path.
"""
from .csa_oracle import (  # noqa: F401
    YaRN, attend, attention_temperature, compress, compress_append, csa_prefill_layer,
    dequantize_fp8_rows, e4m3_encode, e4m3_values, gather_rows, hca_attn, hca_prefill_layer,
    index_scores, index_topk, n_compressed, n_visible, quantize_fp8_rows, rope, rope_freqs,
    rotate_raw, sparse_attn, topk_select, window_tokens)
