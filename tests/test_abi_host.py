"""Host-side checks of the C ABI: the library builds, loads, exports every
symbol include/csa.h declares, and rejects bad arguments before touching a
device.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import sparse_compressed_attention_csa_b200 as csa
from sparse_compressed_attention_csa_b200 import _lib as L
from sparse_compressed_attention_csa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("csa_compress", "csa_index_topk", "csa_sparse_attn", "hca_attn",
              "csa_workspace_size", "csa_status_string", "csa_poll_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_launch_counter_counts_no_rejected_call(lib):
    before = csa.csa_launch_count()
    with pytest.raises(csa.CsaError):
        csa.csa_workspace_size(csa.Params(d=100), csa.CSA_OP_INDEX_TOPK, 1, 1, 10)
    assert csa.csa_launch_count() == before


def test_abi_version_and_status_strings(lib):
    assert lib.csa_abi_version() == 2
    for code, name in L.STATUS.items():
        assert lib.csa_status_string(code).decode() == name


def _status(fn, *args):
    with pytest.raises(csa.CsaError) as ei:
        fn(*args)
    return ei.value.status


def test_query_rows_beyond_one_grid_dimension_are_rejected(lib):
    p = csa.Params()
    assert csa.csa_workspace_size(p, csa.CSA_OP_SPARSE_ATTN, 255, 257, 100) >= 0  # 65535 rows
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_workspace_size(p, csa.CSA_OP_SPARSE_ATTN, 256, 257, 100)
    assert ei.value.status == 3
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_workspace_size(p, csa.CSA_OP_INDEX_TOPK, 0, 1, 100)
    assert ei.value.status == 3


def test_workspace_sizes(lib):
    p = csa.Params()
    n = csa.csa_workspace_size(p, csa.CSA_OP_INDEX_TOPK, 32, 1, 16383)
    assert n >= 32 * 16383 * 4 and n % 256 == 0
    assert csa.csa_workspace_size(p, csa.CSA_OP_COMPRESS, 1, 1, 10) == 0
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_workspace_size(csa.Params(d=100), csa.CSA_OP_INDEX_TOPK, 1, 1, 10)
    assert ei.value.status == 3
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_workspace_size(p, 99, 1, 1, 10)
    assert ei.value.status == 1


def _call_raw(lib, name, *args):
    return getattr(lib, name)(*args)


def test_validation_before_device(lib):
    """Bad parameters, NULL and misaligned pointers return a status; nothing
    reaches a device."""
    p = csa.Params().c()
    pp = ctypes.byref(p)
    P = ctypes.c_void_p
    # NULL params
    assert lib.csa_compress(None, 1, P(16), P(16), 1, 64, P(16), None, None) == 1
    # NULL x
    assert lib.csa_compress(pp, 1, None, P(16), 1, 64, P(16), None, None) == 1
    # misaligned gate
    assert lib.csa_compress(pp, 1, P(16), P(18), 1, 64, P(16), None, None) == 2
    # bad dtype
    assert lib.csa_compress(pp, 7, P(16), P(16), 1, 64, P(16), None, None) == 1
    # unsupported d / odd rope dims / bad width
    for bad in (dict(d=100), dict(rope_dim=63), dict(rope_dim=600), dict(width=0),
                dict(stride=0), dict(window=-1), dict(n_heads=0)):
        q = csa.Params(**bad).c()
        assert lib.csa_compress(ctypes.byref(q), 1, P(16), P(16), 1, 64, P(16), None, None) in (1, 3)
    # extended RoPE (YaRN) without an original context, or with beta_fast <= beta_slow
    for bad in (dict(rope_factor=16.0, rope_orig_ctx=0),
                dict(rope_factor=16.0, rope_orig_ctx=65536, rope_beta_fast=1.0, rope_beta_slow=1.0),
                dict(rope_factor=float("nan"))):
        q = csa.Params(**bad).c()
        assert lib.csa_compress(ctypes.byref(q), 1, P(16), P(16), 1, 64, P(16), None, None) == 1
    # topk out of range
    q = csa.Params(topk=0).c()
    assert lib.csa_topk_select(ctypes.byref(q), P(16), P(16), P(16), 1, 1, 10, P(16), None, 0,
                               None) == 3
    # indexer shape out of range
    q = csa.Params(idx_heads=200, idx_dim=128).c()
    assert lib.csa_index_scores(ctypes.byref(q), 1, P(16), P(16), P(16), P(16), P(16), 1, 1, 10,
                                P(16), None) == 3
    # undersized workspace
    assert lib.csa_index_topk(pp, 1, P(16), P(16), P(16), P(16), P(16), 2, 1, 1000, P(16), P(16),
                              100, None) == 5
    # negative / zero sizes
    assert lib.csa_index_topk(pp, 1, P(16), P(16), P(16), P(16), P(16), 0, 1, 1000, P(16), P(16),
                              1 << 30, None) == 3
    # attention: NULL idx, NULL sink, misaligned out
    assert lib.csa_sparse_attn(pp, 1, P(16), P(16), P(16), None, 10, P(16), P(16), P(16), 4,
                               P(16), 1, 1, P(16), None, 0, None) == 1
    assert lib.csa_sparse_attn(pp, 1, P(16), P(16), P(16), P(16), 10, P(16), P(16), P(16), 4,
                               None, 1, 1, P(16), None, 0, None) == 1
    assert lib.hca_attn(pp, 1, P(16), P(16), P(16), P(16), 10, P(16), P(16), P(16), 4, P(16), 1,
                        1, P(24), None, 0, None) == 2
    assert "aligned" in lib.csa_last_error_detail().decode()


def test_validation_of_the_append_quantize_fp8_and_reuse_calls(lib):
    """The calls beyond the layer's steps reject bad arguments on the host."""
    p = csa.Params().c()
    pp = ctypes.byref(p)
    P = ctypes.c_void_p
    # csa_compress_append: negative sizes, NULL range arrays, misaligned cache
    assert lib.csa_compress_append(pp, 1, P(16), P(16), P(16), 0, 64, P(16), P(16), 8, P(16), 4,
                                   None, None, 0, None) == 3           # B = 0
    assert lib.csa_compress_append(pp, 1, P(16), P(16), P(16), 1, 64, P(16), P(16), -1, P(16), 4,
                                   None, None, 0, None) == 3           # max_new < 0
    assert lib.csa_compress_append(pp, 1, P(16), P(16), P(16), 1, 64, None, P(16), 8, P(16), 4,
                                   None, None, 0, None) == 1           # t_old NULL
    assert lib.csa_compress_append(pp, 1, P(16), P(16), P(16), 1, 64, P(16), P(16), 8, P(24), 4,
                                   None, None, 0, None) == 2           # kv_cmp misaligned
    assert lib.csa_compress_append(pp, 1, P(16), P(16), P(16), 1, 64, P(16), P(16), 8, P(16), 4,
                                   P(16), None, 8, None) == 1          # kv_raw without raw_pos0
    # csa_quantize_fp8: unsupported row width, NULL scales
    assert lib.csa_quantize_fp8(1, P(16), 4, 48, P(16), P(16), None) == 3
    assert lib.csa_quantize_fp8(1, P(16), 4, 512, P(16), None, None) == 1
    assert lib.csa_quantize_fp8(1, P(16), 0, 512, None, None, None) == 0  # nothing to do
    # FP8 attention: a shape off the tensor-core path; NULL scales
    q = csa.Params(n_heads=64).c()
    assert lib.csa_sparse_attn_fp8(ctypes.byref(q), P(16), P(16), P(16), P(16), P(16), 10, P(16),
                                   P(16), P(16), P(16), 4, P(16), 1, 1, P(16), None, 0, None) == 3
    assert lib.csa_sparse_attn_fp8(pp, P(16), P(16), P(16), None, P(16), 10, P(16), P(16), P(16),
                                   P(16), 4, P(16), 1, 1, P(16), None, 0, None) == 1
    assert lib.hca_attn_fp8(pp, P(16), P(16), P(16), P(16), P(16), 10, P(16), None, P(16), P(16),
                            4, P(16), 1, 1, P(16), None, 0, None) == 1
    # csa_reuse_attn: no layers, or layers x B x Tq beyond one grid dimension
    assert lib.csa_reuse_attn(pp, 1, 0, P(16), P(16), P(16), P(16), 10, P(16), P(16), P(16), 4,
                              P(16), 1, 1, P(16), None, 0, None) == 3
    assert lib.csa_reuse_attn(pp, 1, 2, P(16), P(16), P(16), P(16), 10, P(16), P(16), P(16), 4,
                              P(16), 40000, 1, P(16), None, 0, None) == 3


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(ImportError):
        L.lib()
