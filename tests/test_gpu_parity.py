"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bit-exact top-k indices (and indexer scores, which are exact integers times
powers of two); outputs within max-abs / relative-L2 bounds (bf16 2e-2 /
5e-3, fp32 1e-5).  Every workload runs at its full size in the launch
configuration the benchmark times; the oracle checks every sequence of the
decode workloads and a stratified sample of the prefill queries.  Smaller
cases cover several tiles with ragged tails and the edge cases.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_close, dev, f64, host64, params_of, run_decode, run_hca,
                      run_prefill, theta_of)
from sparse_compressed_attention_csa_b200 import (CSA_OP_SPARSE_ATTN, CSA_OP_TOPK_SELECT,
                                                  CsaError, Params,
                                                  csa_compress, csa_workspace_size,
                                                  csa_index_scores, csa_poll_device_error,
                                                  csa_sparse_attn, csa_topk_select)
from sparse_compressed_attention_csa_b200 import layer
from sparse_compressed_attention_csa_b200 import workloads as W
from sparse_compressed_attention_csa_b200.workloads import bits_to_f32, to_f64

pytestmark = pytest.mark.gpu


def _vals(a):
    """Generated array as real values (fp32 view of bf16 bits)."""
    return bits_to_f32(a) if a.dtype == np.uint16 else a


# ------------------------------------------------------------------ oracle drivers
def oracle_decode(wl, data, seqs):
    idx_all, out_all = [], []
    for b in seqs:
        qp = data["q_pos"][b]
        idx = oracle.index_topk(f64(data, "q_idx", b), data["w"][b], f64(data, "k_idx", b), qp,
                                int(data["n_cmp"][b]), wl.width, wl.stride, wl.topk)
        out = oracle.sparse_attn(f64(data, "q", b), qp, _vals(data["kv_cmp"][b]), idx,
                                 _vals(data["kv_raw"][b]), int(data["raw_pos0"][b]),
                                 int(data["n_raw"][b]), data["sink"], wl.scale, wl.window,
                                 wl.rope_dim, theta_of(wl))
        idx_all.append(idx)
        out_all.append(out)
    return np.stack(idx_all), np.stack(out_all)


def check_decode(wl, seqs=None):
    data = W.generate(wl)
    idx, out = run_decode(wl, data)
    seqs = list(range(wl.B)) if seqs is None else seqs
    idx_o, out_o = oracle_decode(wl, data, seqs)
    got_idx = idx.cpu().numpy()[seqs]
    assert np.array_equal(got_idx, idx_o), "top-k indices differ"
    assert_close(host64(out)[seqs], out_o, wl.dtype, wl.name)


def check_hca(wl, seqs=None):
    data = W.generate(wl)
    out = run_hca(wl, data)
    seqs = list(range(wl.B)) if seqs is None else seqs
    got = host64(out)[seqs]
    want = np.stack([oracle.hca_attn(f64(data, "q", b), data["q_pos"][b],
                                     _vals(data["kv_cmp"][b]), int(data["n_cmp"][b]),
                                     _vals(data["kv_raw"][b]), int(data["raw_pos0"][b]),
                                     int(data["n_raw"][b]), data["sink"], wl.scale, wl.window,
                                     wl.width, wl.stride, wl.rope_dim, theta_of(wl))
                     for b in seqs])
    assert_close(got, want, wl.dtype, wl.name)


def check_prefill(wl, rows=None):
    data = W.generate(wl)
    kv_cmp, kv_raw, idx, out = run_prefill(wl, data)
    T = wl.T
    rows = np.arange(T) if rows is None else np.asarray(rows)
    for b in range(wl.B):
        x, g = f64(data, "x", b), f64(data, "g", b)
        cmp_o = oracle.compress(x, g, wl.width, wl.stride, wl.rope_dim, theta_of(wl), wl.pos_offset)
        assert_close(host64(kv_cmp[b]), cmp_o, wl.dtype, "compressed entries")
        raw_o = oracle.rotate_raw(x, 0, wl.rope_dim, theta_of(wl))
        assert_close(host64(kv_raw[b]), raw_o, wl.dtype, "rotated raw rows")
        qp = data["q_pos"][b]
        idx_o = oracle.index_topk(_vals(data["q_idx"][b]), data["w"][b], f64(data, "k_idx", b),
                                  qp, cmp_o.shape[0], wl.width, wl.stride, wl.topk, rows)
        assert np.array_equal(idx[b].cpu().numpy()[rows], idx_o), "top-k indices differ"
        out_o = oracle.sparse_attn(to_f64(data["q"][b][rows]), qp[rows], cmp_o, idx_o, raw_o, 0,
                                   T, data["sink"], wl.scale, wl.window, wl.rope_dim, theta_of(wl))
        sel = torch.as_tensor(rows, device=out.device)
        assert_close(host64(out[b][sel]), out_o, wl.dtype, wl.name)


def check_hca_prefill(wl, rows=None):
    data = W.generate(wl)
    p = params_of(wl)
    kv_cmp, kv_raw, out = layer.hca_prefill(p, dev(data["x"]), dev(data["g"]), dev(data["q"]),
                                            dev(data["sink"]))
    torch.cuda.synchronize()
    T = wl.T
    rows = np.arange(T) if rows is None else np.asarray(rows)
    th = theta_of(wl)
    for b in range(wl.B):
        x, g = f64(data, "x", b), f64(data, "g", b)
        cmp_o = oracle.compress(x, g, wl.width, wl.stride, wl.rope_dim, th, wl.pos_offset)
        assert_close(host64(kv_cmp[b]), cmp_o, wl.dtype, "HCA entries")
        raw_o = oracle.rotate_raw(x, 0, wl.rope_dim, th)
        assert_close(host64(kv_raw[b]), raw_o, wl.dtype, "HCA raw rows")
        # the oracle's HCA prefill restricted to the sampled query rows
        out_o = oracle.hca_attn(to_f64(data["q"][b][rows]), rows, cmp_o, cmp_o.shape[0], raw_o,
                                0, T, data["sink"], wl.scale, wl.window, wl.width, wl.stride,
                                wl.rope_dim, th)
        sel = torch.as_tensor(rows, device=out.device)
        assert_close(host64(out[b][sel]), out_o, wl.dtype, wl.name)


# ------------------------------------------------------------------ the five workloads
def test_tiny_f32_full_layer():
    check_prefill(W.TINY_F32)


def test_csa_decode_64k_bs32():
    check_decode(W.CSA_DECODE_64K)


def test_csa_decode_1m_bs4():
    check_decode(W.CSA_DECODE_1M)


def test_hca_decode_128k_bs16():
    check_hca(W.HCA_DECODE_128K)


def test_csa_prefill_8k():
    # the first rows (nothing or few entries visible), a block boundary, the
    # last rows, and 256 rows drawn uniformly: every query token runs its own
    # CTA pairs, so the sample covers 256 independent launches' worth of
    # work at full size
    rng = np.random.default_rng(1234)
    rows = np.unique(np.concatenate([np.arange(0, 16), np.arange(4095, 4104),
                                     np.arange(8176, 8192), rng.integers(0, 8192, 256)]))
    assert rows.size >= 256
    check_prefill(W.CSA_PREFILL_8K, rows)


# ------------------------------------------------------------------ smaller cases
def test_hca_prefill_8k():
    # every entry and raw row; query rows: the first 300 (0, 1 and 2 entries
    # visible, the window filling up) and a stride through the rest
    rows = np.unique(np.concatenate([np.arange(300), np.arange(300, 8192, 37), [8191]]))
    check_hca_prefill(W.HCA_PREFILL_8K, rows)


def test_hca_prefill_ragged_small():
    # T = 1000: 7 entries, a partial last block of 104 tokens; two sequences
    check_hca_prefill(W.HCA_PREFILL_8K.replace(B=2, T=1000, seed=48))


def test_decode_ragged_tiles():
    # N = 1249 (ragged), selection active (n_vis > k), raw window 128
    check_decode(W.CSA_DECODE_64K.replace(B=3, T=5003, seed=21))


def test_decode_fewer_visible_than_k():
    check_decode(W.CSA_DECODE_64K.replace(B=2, T=2100, seed=22))  # N = 524 < 1024


def test_decode_running_max_moves_for_some_heads_only():
    # the last selected entry of each sequence (the list's last tile: window
    # rows come first, entries after, in index order) set to 14 x the unit
    # direction of the query of one head per warp (heads 3, 40, 77, 110;
    # non-rotated dims only): those heads see a logit of about 13 on it,
    # above their running maximum by more than the lazy-rescale threshold
    # (2^8), the other heads a small one, so the lanes of each softmax warp
    # disagree on rescaling O in a late tile.  The row's values stay of order
    # one (the tolerance is absolute).
    wl = W.CSA_DECODE_64K.replace(B=2, T=5003, seed=47)
    data = W.generate(wl)
    idx_o = np.stack([oracle.index_topk(f64(data, "q_idx", b), data["w"][b], f64(data, "k_idx", b),
                                        data["q_pos"][b], int(data["n_cmp"][b]), wl.width,
                                        wl.stride, wl.topk)[0] for b in range(wl.B)])
    cmp = bits_to_f32(data["kv_cmp"]).copy()
    q = bits_to_f32(data["q"]).astype(np.float64)  # [B, 1, H, d]
    nr = wl.d - wl.rope_dim
    for b in range(wl.B):
        row = np.zeros(wl.d)
        for h in (3, 40, 77, 110):
            u = q[b, 0, h, :nr]
            row[:nr] += 14.0 * u / np.linalg.norm(u)
        cmp[b, idx_o[b].max()] = row
    data["kv_cmp"] = W.bf16_bits(cmp)
    idx, out = run_decode(wl, data)
    idx_w, out_o = oracle_decode(wl, data, [0, 1])
    assert np.array_equal(idx.cpu().numpy(), idx_w), "top-k indices differ"
    assert_close(host64(out), out_o, wl.dtype, "decode with an aligned selected entry")


def test_decode_extended_rope_past_the_original_context():
    # theta 160,000 with YaRN (factor 16 over 65,536 tokens) on queries at
    # position 131,071: q and the output's inverse rotation use the YaRN
    # frequencies, the logits the YaRN temperature
    check_decode(W.CSA_DECODE_YARN.replace(B=4, seed=44))


def test_prefill_extended_rope_small_original_context():
    # the same extension with an original context of 512 tokens, so that a
    # 1,500-token prefill runs past it in the pooled entries, the raw rows
    # and the queries alike; ragged tail, every query row checked
    wl = W.CSA_PREFILL_8K.replace(T=1500, topk=128, seed=45, theta=160000.0, rope_factor=4.0,
                                  rope_orig_ctx=512)
    check_prefill(wl, rows=np.arange(0, 1500, 3))


def test_csa2_full_and_reuse_layers():
    # 2 -> 1 pooling, top-512, YaRN; the Reuse layers attend with their own
    # queries and sinks over the Full layer's entries and selection
    wl = W.CSA2_DECODE.replace(B=3, T=20001, reuse_layers=3, seed=46)
    data = W.generate(wl)
    idx, out = run_decode(wl, data)
    seqs = list(range(wl.B))
    idx_o, out_o = oracle_decode(wl, data, seqs)
    assert np.array_equal(idx.cpu().numpy(), idx_o), "top-k indices differ"
    assert_close(host64(out), out_o, wl.dtype, wl.name)
    p = params_of(wl)
    t = {k: dev(data[k]) for k in ("q_pos", "kv_cmp", "kv_raw", "raw_pos0", "n_raw")}
    # every Reuse layer in one call, and layer 1 alone
    o_all = layer.reuse_attn(p, dev(data["q_reuse"]), t["q_pos"], t["kv_cmp"], idx, t["kv_raw"],
                             t["raw_pos0"], t["n_raw"], dev(data["sink_reuse"]))
    o_one = layer.reuse_attn(p, dev(data["q_reuse"][1]), t["q_pos"], t["kv_cmp"], idx,
                             t["kv_raw"], t["raw_pos0"], t["n_raw"], dev(data["sink_reuse"][1]))
    torch.cuda.synchronize()
    for r in range(wl.reuse_layers):
        want = np.stack([oracle.sparse_attn(
            f64(data, "q_reuse", r, b),
            data["q_pos"][b], _vals(data["kv_cmp"][b]), idx_o[b], _vals(data["kv_raw"][b]),
            int(data["raw_pos0"][b]), int(data["n_raw"][b]), data["sink_reuse"][r], wl.scale,
            wl.window, wl.rope_dim, theta_of(wl)) for b in seqs])
        assert_close(host64(o_all[r]), want, wl.dtype, f"{wl.name} reuse layer {r}")
        if r == 1:
            assert_close(host64(o_one), want, wl.dtype, f"{wl.name} reuse layer 1 alone")


def test_decode_context_too_short_for_any_entry():
    # T = 5 < width: no compressed entry, so no scores, every index -1 and the
    # attention runs over the window and the sink only
    check_decode(W.CSA_DECODE_64K.replace(B=2, T=5, seed=33))


def test_decode_rows_at_the_tensor_core_cap_and_beyond():
    # 1,900 selected + 128 window rows fill the tensor-core kernel's row list;
    # 1,950 + 128 go past it and take the generic kernel
    check_decode(W.CSA_DECODE_64K.replace(B=2, T=10000, topk=1900, seed=34))
    check_decode(W.CSA_DECODE_64K.replace(B=2, T=10000, topk=1950, seed=35))


def test_prefill_ragged_small():
    check_prefill(W.CSA_PREFILL_8K.replace(T=777, topk=64, seed=23))


def test_prefill_small_heads_f32():
    check_prefill(W.TINY_F32.replace(T=203, n_heads=3, topk=7, window=5, seed=24, pos_offset=2))


def test_hca_ragged_and_early_queries():
    check_hca(W.HCA_DECODE_128K.replace(B=3, T=1000, seed=25))   # N = 7
    check_hca(W.HCA_DECODE_128K.replace(B=2, T=100, seed=26))    # N = 0: window + sink only
    check_hca(W.HCA_DECODE_128K.replace(B=2, T=3, seed=27))      # one split holds no rows


def test_compress_hca_width_bf16_and_f32():
    for dtype in ("bf16", "f32"):
        wl = W.CSA_PREFILL_8K.replace(dtype=dtype, T=1000, width=128, stride=128, seed=27)
        data = W.generate(wl)
        p = params_of(wl)
        x, g = dev(data["x"]), dev(data["g"])
        N = wl.n_cmp
        kv = torch.empty((1, N, wl.d), dtype=x.dtype, device="cuda")
        csa_compress(p, x, g, kv)
        torch.cuda.synchronize()
        want = oracle.compress(f64(data, "x", 0), f64(data, "g", 0), 128, 128, wl.rope_dim,
                               theta_of(wl))
        assert_close(host64(kv[0]), want, dtype, f"hca compress {dtype}")


def test_index_scores_bit_exact():
    wl = W.CSA_PREFILL_8K.replace(T=1503, seed=28)
    data = W.generate(wl)
    p = params_of(wl)
    t = {k: dev(data[k]) for k in ("q_idx", "w", "k_idx", "q_pos", "n_cmp")}
    sc = torch.full((1, wl.T, wl.n_cmp), float("nan"), dtype=torch.float32, device="cuda")
    csa_index_scores(p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], sc)
    torch.cuda.synchronize()
    got = sc[0].cpu().numpy().astype(np.float64)
    want = oracle.index_scores(f64(data, "q_idx", 0), data["w"][0], f64(data, "k_idx", 0))
    for tq in range(0, wl.T, 7):
        nv = oracle.n_visible(tq, wl.n_cmp, wl.width, wl.stride)
        assert np.array_equal(got[tq, :nv], want[tq, :nv]), tq


def test_index_scores_decode_ragged_visibility():
    # one query per sequence at different positions: the decode indexer skips
    # tiles past each sequence's visible entries and switches query blocks
    # where a CTA's range of tiles crosses a sequence boundary
    wl = W.CSA_DECODE_64K.replace(B=7, T=20000, seed=32)
    data = W.generate(wl)
    data["q_pos"] = np.array([[19999], [5000], [129], [7], [3000], [19998], [0]], dtype=np.int32)
    p = params_of(wl)
    t = {k: dev(data[k]) for k in ("q_idx", "w", "k_idx", "q_pos", "n_cmp")}
    sc = torch.full((wl.B, 1, wl.n_cmp), float("nan"), dtype=torch.float32, device="cuda")
    csa_index_scores(p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], sc)
    torch.cuda.synchronize()
    got = sc.cpu().numpy().astype(np.float64)
    for b in range(wl.B):
        nv = oracle.n_visible(int(data["q_pos"][b, 0]), wl.n_cmp, wl.width, wl.stride)
        want = oracle.index_scores(f64(data, "q_idx", b), data["w"][b], f64(data, "k_idx", b))
        assert np.array_equal(got[b, 0, :nv], want[0, :nv]), b
        assert np.all(np.isnan(got[b, 0, nv:])), b  # nothing written past the visible entries


def _adversarial_rows(rng, n):
    return [
        np.zeros(n),                                        # all tied
        np.where(rng.random(n) < 0.5, 0.0, -0.0),           # signed zeros tie
        rng.integers(0, 3, n).astype(np.float64),           # few distinct values
        -rng.random(n),                                     # negatives
        rng.standard_normal(n) * 1e-30,                     # tiny magnitudes
        np.concatenate([np.full(n // 2, 7.0), rng.random(n - n // 2)]),
        rng.standard_normal(n).astype(np.float32).astype(np.float64),
    ]


# (entries, k, rows, visible): few rows of up to 32768 entries take a cluster
# of 4096-entry CTAs per row, few rows of up to 262144 a cluster of up to 16
# CTAs of 16384; otherwise one block per row up to 16384 entries, else
# chunks of 16384 and a merge block of 4096, 8192 or 16384 candidates
@pytest.mark.parametrize("n,k,rows,visible", [
    (5000, 1024, 7, None),     # cluster of 2
    (9000, 64, 3, None),       # cluster of 3
    (16383, 1024, 5, None),    # cluster of 4
    (30000, 1024, 7, None),    # cluster of 8
    (20000, 1024, 3, 700),     # cluster of 5, fewer visible than k
    (5000, 1024, 84, None),    # one 16384-entry block per row
    (1500, 64, 20, None),      # one 2048-entry block per row
    (32767, 1024, 32, None),   # 32 rows x 8 CTAs of 4096 do not fit: cluster of 2 of 16384
    (40000, 1024, 7, None),    # cluster of 3 CTAs of 16384 entries
    (70000, 3000, 3, None),    # cluster of 5 of 16384, k = 3000
    (262143, 1024, 4, None),   # cluster of 16 of 16384 (the 1M-context rows)
    (200000, 1024, 3, 150001), # cluster of 13, fewer visible than the CTAs hold
    (40000, 1024, 60, None),   # 180 CTAs for a cluster each: 3 chunks, merge of 3072
    (70000, 1024, 40, None),   # 5 chunks, merge of 5120
])
def test_topk_select_adversarial_scores(n, k, rows, visible):
    rng = np.random.default_rng(29 + n + k + rows)
    base = _adversarial_rows(rng, n)
    scores = np.stack([base[r % len(base)] for r in range(rows)]).astype(np.float32)[:, None, :]
    B = scores.shape[0]
    p = Params(topk=k, width=8, stride=4)
    nv = n if visible is None else visible
    q_pos = np.full((B, 1), 4 * (nv - 1) + 7, dtype=np.int32)   # entries 0 .. nv-1 visible
    n_cmp = np.full((B,), n, dtype=np.int32)
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    nb = csa_workspace_size(p, CSA_OP_TOPK_SELECT, B, 1, n)
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda")
    csa_topk_select(p, dev(scores), dev(q_pos), dev(n_cmp), idx, ws)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    for b in range(B):
        want = oracle.topk_select(scores[b, 0].astype(np.float64), nv, k)
        assert np.array_equal(got[b, 0], want), b


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


@pytest.mark.parametrize("case", ["decode_64k", "decode_long_rows", "hca_decode", "prefill"])
def test_deterministic_repeat(case):
    # ten runs on the same inputs give bitwise-identical outputs and the same
    # top-k: the pair's partial-logit exchange, the cluster top-k's exchanges
    # and the split-KV merge all combine in a fixed order
    wl, run = {
        "decode_64k": (W.CSA_DECODE_64K.replace(B=2, T=9000, seed=30), run_decode),
        # rows of 100,000 entries: the wide top-k cluster and many KV splits
        "decode_long_rows": (W.CSA_DECODE_1M.replace(B=2, T=4 * 100000 + 4, seed=32), run_decode),
        "hca_decode": (W.HCA_DECODE_128K.replace(B=3, T=128 * 700 + 5, seed=33), run_hca),
        "prefill": (W.CSA_PREFILL_8K.replace(T=1203, topk=256, seed=34), run_prefill),
    }[case]
    data = W.generate(wl)

    def once():
        r = run(wl, data)
        return [_bits(x) for x in (r if isinstance(r, tuple) else (r,))]

    first = once()
    for _ in range(9):
        for a, b in zip(first, once()):
            assert torch.equal(a, b), case


def test_device_bounds_error_is_reported():
    """An index past the cache is skipped and reported, not dereferenced."""
    wl = W.CSA_DECODE_64K.replace(B=1, T=600, seed=31, topk=16)
    data = W.generate(wl)
    p = params_of(wl)
    t = {k: dev(v) for k, v in data.items()}
    idx = torch.arange(16, dtype=torch.int32, device="cuda").view(1, 1, 16).contiguous()
    idx[0, 0, 5] = wl.n_cmp + 1000
    out = torch.empty_like(t["q"])
    nb = csa_workspace_size(p, CSA_OP_SPARSE_ATTN, 1, 1, t["kv_cmp"].shape[1])
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    csa_poll_device_error()
    csa_sparse_attn(p, t["q"], t["q_pos"], t["kv_cmp"], idx, t["kv_raw"], t["raw_pos0"],
                    t["n_raw"], t["sink"], out, ws)
    with pytest.raises(CsaError) as ei:
        csa_poll_device_error()
    assert ei.value.status == 8
    csa_poll_device_error()  # cleared
