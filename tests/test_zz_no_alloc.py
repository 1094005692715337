"""The indexer + top-k entry point that allocates nothing.

csa_index_topk_noalloc serves callers that cannot call cudaMalloc or hand
the library a workspace (hosts that pass only input and output buffers,
engines whose allocator already owns all device memory, loops that cannot
afford cudaMalloc's device-wide synchronization).  It keeps its scores in a
fixed array built into the library.  This test checks, through the C ABI,
that two calls in a row give exactly the indices of csa_index_topk, which
uses a caller workspace (also for rows long enough to need the top-k
candidate lists kept in the array), and that sizes beyond the array are
rejected.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import pytest
import torch

from gpu_util import dev, params_of
from sparse_compressed_attention_csa_b200 import (CSA_OP_INDEX_TOPK, CsaError, csa_index_topk,
                                                  csa_index_topk_noalloc, csa_poll_device_error,
                                                  csa_workspace_size)
from sparse_compressed_attention_csa_b200 import workloads as W

pytestmark = pytest.mark.gpu


_KEYS = ("q_idx", "w", "k_idx", "q_pos", "n_cmp")


def _inputs(wl):
    d = W.generate(wl, keys=_KEYS)
    return {k: dev(d[k]) for k in _KEYS}


def _with_workspace(p, t):
    B, Tq = t["q_pos"].shape
    n_max = t["k_idx"].shape[1]
    nb = csa_workspace_size(p, CSA_OP_INDEX_TOPK, B, Tq, n_max)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    idx = torch.empty((B, Tq, p.topk), dtype=torch.int32, device="cuda")
    csa_index_topk(p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], idx, ws)
    return idx


def _no_alloc(p, t):
    B, Tq = t["q_pos"].shape
    idx = torch.full((B, Tq, p.topk), -7, dtype=torch.int32, device="cuda")
    csa_index_topk_noalloc(p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], idx)
    return idx


def test_no_alloc_matches_workspace_call_twice_in_a_row():
    # call 1: the 64K-context decode batch (32 x 16,383 scores fill 1/4 of
    # the array); call 2: a causal prefill whose scores overwrite part of it
    first = W.CSA_DECODE_64K
    second = W.CSA_PREFILL_8K.replace(T=1203, topk=256, seed=41)
    for wl in (first, second):
        p = params_of(wl)
        t = _inputs(wl)
        want = _with_workspace(p, t)
        got = _no_alloc(p, t)
        torch.cuda.synchronize()
        csa_poll_device_error()
        assert torch.equal(got, want), wl.name
        assert int((got >= 0).sum()) > 0


def test_no_alloc_long_rows_use_candidate_lists_from_its_array():
    # 50 rows of 33,000 entries: too long for one top-k block and too many
    # rows for a cluster of CTAs each, so each row is cut into chunks whose
    # candidate lists sit in the array after the scores
    wl = W.CSA_DECODE_1M.replace(B=50, T=4 * 33000 + 4, seed=43)
    p = params_of(wl)
    t = _inputs(wl)
    want = _with_workspace(p, t)
    got = _no_alloc(p, t)
    torch.cuda.synchronize()
    csa_poll_device_error()
    assert torch.equal(got, want)
    assert int((got >= 0).sum()) == 50 * p.topk


def test_no_alloc_rejects_sizes_beyond_its_array():
    wl = W.CSA_DECODE_64K.replace(B=2, T=4 * 4096 + 4)   # small real inputs
    p = params_of(wl)
    t = _inputs(wl)
    big_n = (1 << 21) // 2 + 1                              # 2 * n_max > 2^21 scores
    k_big = torch.zeros((2, big_n, wl.idx_dim), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((2, 1, p.topk), dtype=torch.int32, device="cuda")
    with pytest.raises(CsaError) as ei:
        csa_index_topk_noalloc(p, t["q_idx"], t["w"], k_big, t["q_pos"], t["n_cmp"], idx)
    assert ei.value.status == 3
    assert "no-alloc scratch" in str(ei.value) and "bytes" in str(ei.value)
