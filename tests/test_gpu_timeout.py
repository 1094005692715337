"""A bounded device-side wait that runs out: the kernel records
CSA_ERR_DEVICE_TIMEOUT in the device error word, drains what it issued,
frees its tensor memory and returns, and the context stays usable.

The wait limit is made tiny with csa_set_wait_limit_ns, so the first wait
of the tensor-core indexer that is not satisfied at once gives up (its
tiles take microseconds to arrive).  No fault, trap or endless loop is
involved: every wait in the kernel is bounded, the wind-down waits too.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import dev, f64, params_of
from sparse_compressed_attention_csa_b200 import (CsaError, csa_index_scores,
                                                  csa_poll_device_error, csa_set_wait_limit_ns)
from sparse_compressed_attention_csa_b200 import workloads as W

pytestmark = pytest.mark.gpu

CSA_ERR_DEVICE_TIMEOUT = 7


def _scores(p, t, wl):
    sc = torch.full((wl.B, 1, wl.n_cmp), float("nan"), dtype=torch.float32, device="cuda")
    csa_index_scores(p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], sc)
    return sc


def test_wait_runs_out_then_next_call_matches_the_oracle():
    # decode indexer on the tensor-core path (64 x 128 bf16), 2 x 1,249 entries
    wl = W.CSA_DECODE_64K.replace(B=2, T=5003, seed=41)
    data = W.generate(wl)
    p = params_of(wl)
    t = {k: dev(data[k]) for k in ("q_idx", "w", "k_idx", "q_pos", "n_cmp")}
    csa_poll_device_error()  # starts clean
    csa_set_wait_limit_ns(1)
    try:
        _scores(p, t, wl)
        with pytest.raises(CsaError) as err:
            csa_poll_device_error()
        assert err.value.status == CSA_ERR_DEVICE_TIMEOUT
    finally:
        csa_set_wait_limit_ns(0)  # back to the default limit
    csa_poll_device_error()  # the error word was cleared by the read above
    sc = _scores(p, t, wl)
    csa_poll_device_error()
    got = sc[:, 0].cpu().numpy().astype(np.float64)
    for b in range(wl.B):
        want = oracle.index_scores(f64(data, "q_idx", b), data["w"][b], f64(data, "k_idx", b))[0]
        nv = oracle.n_visible(int(data["q_pos"][b][0]), wl.n_cmp, wl.width, wl.stride)
        assert np.array_equal(got[b, :nv], want[:nv]), b


def test_attention_wait_runs_out_then_next_call_matches_the_oracle():
    # the CTA-pair attention kernel (decode, 2 sequences, top-1,024 of 1,249
    # entries + window: several tiles per split, split-KV merge): with a 1 ns
    # limit its first unsatisfied wait gives up; every role winds down
    # (drains its copies, MMAs and partner stores), the call records the
    # timeout with the line of the wait, and the next call is exact again
    from sparse_compressed_attention_csa_b200 import (CSA_OP_SPARSE_ATTN,
                                                      csa_last_device_error_site, csa_sparse_attn,
                                                      csa_workspace_size)
    wl = W.CSA_DECODE_64K.replace(B=2, T=5003, seed=42)
    data = W.generate(wl)
    p = params_of(wl)
    t = {k: dev(data[k]) for k in ("q", "q_pos", "kv_cmp", "kv_raw", "raw_pos0", "n_raw", "sink")}
    idx_o = np.stack([oracle.index_topk(f64(data, "q_idx", b), data["w"][b], f64(data, "k_idx", b),
                                        data["q_pos"][b], int(data["n_cmp"][b]), wl.width,
                                        wl.stride, wl.topk) for b in range(wl.B)])
    idx = torch.from_numpy(idx_o.astype(np.int32)).cuda()
    nb = csa_workspace_size(p, CSA_OP_SPARSE_ATTN, wl.B, 1, wl.n_cmp)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(t["q"])

    def attend():
        csa_sparse_attn(p, t["q"], t["q_pos"], t["kv_cmp"], idx, t["kv_raw"], t["raw_pos0"],
                        t["n_raw"], t["sink"], out, ws)

    csa_poll_device_error()
    csa_set_wait_limit_ns(1)
    try:
        attend()
        with pytest.raises(CsaError) as err:
            csa_poll_device_error()
        assert err.value.status == CSA_ERR_DEVICE_TIMEOUT
        assert csa_last_device_error_site() > 0
    finally:
        csa_set_wait_limit_ns(0)
    csa_poll_device_error()
    attend()
    csa_poll_device_error()
    got = out.float().cpu().numpy().astype(np.float64)
    for b in range(wl.B):
        want = oracle.sparse_attn(f64(data, "q", b), data["q_pos"][b],
                                  W.bits_to_f32(data["kv_cmp"][b]), idx_o[b],
                                  W.bits_to_f32(data["kv_raw"][b]), int(data["raw_pos0"][b]),
                                  int(data["n_raw"][b]), data["sink"], wl.scale, wl.window,
                                  wl.rope_dim, wl.theta)
        err_abs = np.max(np.abs(got[b] - want))
        assert err_abs <= 2e-2, (b, err_abs)
