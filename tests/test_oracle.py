"""Pins of the fp64 oracle against what the pages and mathematics fix.

None of these tests retypes the oracle's formulas: they use closed forms,
invariants, a library routine the method reduces to (torch SDPA in float64),
an independent pure-Python brute force (tests/brute.py) and the entry counts
the workloads state (tests/golden/entry_counts.txt).
"""
import math
import os

import numpy as np
import pytest
import torch

import brute
import oracle
from oracle import csa_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
THETA = 10000.0


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- counts
def test_entry_counts_match_stated_workloads():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "entry_counts.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 6
    for T, w, s, n in (map(int, r) for r in rows):
        assert oracle.n_compressed(T, w, s) == n


def test_visibility_counts():
    # decode query at the last context token sees every pooled entry
    assert oracle.n_visible(65535, 16383, 8, 4) == 16383
    assert oracle.n_visible(1048575, 262143, 8, 4) == 262143
    assert oracle.n_visible(131071, 1024, 128, 128) == 1024
    # an entry is visible once its last (8th) token has been seen
    assert oracle.n_visible(6, 100, 8, 4) == 0
    assert oracle.n_visible(7, 100, 8, 4) == 1
    assert oracle.n_visible(10, 100, 8, 4) == 1
    assert oracle.n_visible(11, 100, 8, 4) == 2
    for t in range(0, 80):
        assert oracle.n_visible(t, 1000, 8, 4) == len(brute.visible(t, 1000, 8, 4))


def test_window_tokens():
    assert list(oracle.window_tokens(5, 16, 0, 256)) == list(range(0, 6))
    assert list(oracle.window_tokens(300, 16, 0, 1000)) == list(range(285, 301))
    assert list(oracle.window_tokens(65535, 128, 65408, 128)) == list(range(65408, 65536))
    for t in (0, 3, 17, 40):
        assert list(oracle.window_tokens(t, 16, 10, 20)) == brute.window(t, 16, 10, 20)


# ---------------------------------------------------------------- RoPE
def test_rope_is_complex_rotation():
    x = _rng(0).standard_normal((5, 32))
    pos = np.array([0, 1, 7, 1000, 65535])
    r = 16
    got = oracle.rope(x, pos, r, THETA)
    assert np.array_equal(got[:, :16], x[:, :16])  # leading dims untouched
    i = np.arange(r // 2)
    z = (x[:, 16::2] + 1j * x[:, 17::2]) * np.exp(1j * np.outer(pos, THETA ** (-2.0 * i / r)))
    np.testing.assert_allclose(got[:, 16::2], z.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[:, 17::2], z.imag, rtol=0, atol=1e-12)


def test_rope_relative_distance_and_inverse():
    rng = _rng(1)
    a, b = rng.standard_normal(64), rng.standard_normal(64)
    dots = [oracle.rope(a, p, 64, THETA) @ oracle.rope(b, p - 37, 64, THETA)
            for p in (40, 1000, 123456)]
    np.testing.assert_allclose(dots, dots[0], rtol=0, atol=1e-9)
    back = oracle.rope(oracle.rope(a, 777, 64, THETA), -777, 64, THETA)
    np.testing.assert_allclose(back, a, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- compress
def test_uniform_gates_make_exact_mean_pooling():
    rng = _rng(2)
    x = rng.standard_normal((40, 24))
    g = np.full((40, 24), 0.37)
    e = oracle.compress(x, g, 8, 4, 0, THETA)
    assert e.shape == (9, 24)
    for j in range(9):
        np.testing.assert_allclose(e[j], x[4 * j:4 * j + 8].mean(axis=0), rtol=0, atol=1e-14)


def test_dominant_gate_copies_one_tap():
    rng = _rng(3)
    x = rng.standard_normal((24, 16))
    g = np.zeros((24, 16))
    g[np.arange(24) % 4 == 1] = 800.0  # tap u=1 of every entry dominates
    e = oracle.compress(x, g, 8, 4, 0, THETA)
    # taps 1 and 5 of each window both carry the large logit: equal halves
    for j in range(e.shape[0]):
        np.testing.assert_allclose(e[j], 0.5 * (x[4 * j + 1] + x[4 * j + 5]), atol=1e-12)


def test_compress_matches_brute_force():
    rng = _rng(4)
    for (T, d, w, s, r) in ((19, 16, 8, 4, 8), (20, 8, 4, 4, 4), (9, 6, 2, 2, 2)):
        x, g = rng.standard_normal((T, d)), rng.standard_normal((T, d))
        got = oracle.compress(x, g, w, s, r, THETA, pos_offset=3)
        ref = np.array(brute.compress(x.tolist(), g.tolist(), w, s, r, THETA, 3))
        assert got.shape == ref.shape
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- indexer
def test_index_scores_integer_exact_and_brute():
    rng = _rng(5)
    q = rng.integers(-8, 9, size=(3, 4, 16)).astype(np.float64)
    k = rng.integers(-8, 9, size=(21, 16)).astype(np.float64)
    w = np.exp2(rng.integers(-2, 3, size=(3, 4))).astype(np.float64)
    got = oracle.index_scores(q, w, k)
    for t in range(3):
        ref = brute.scores(q[t].tolist(), w[t].tolist(), k.tolist())
        assert got[t].tolist() == ref  # integers times powers of two: exact
        # exact integer arithmetic, times 4 to clear the 2^-2 weights
        exact = [sum(int(w[t, h] * 4) * max(0, int(q[t, h] @ k[j])) for h in range(4))
                 for j in range(21)]
        assert (got[t] * 4).astype(np.int64).tolist() == exact


def test_topk_ties_and_order():
    rng = _rng(6)
    for trial in range(30):
        n = int(rng.integers(1, 60))
        s = rng.integers(0, 5, size=n).astype(np.float64)  # many ties
        k = int(rng.integers(1, 20))
        nv = int(rng.integers(0, n + 1))
        got = oracle.topk_select(s, nv, k)
        assert got.tolist() == brute.topk(s.tolist(), nv, k)


def test_topk_fewer_visible_keeps_all_and_pads():
    s = np.array([5.0, 1.0, 9.0, 2.0])
    assert oracle.topk_select(s, 3, 8).tolist() == [0, 1, 2, -1, -1, -1, -1, -1]
    assert oracle.topk_select(s, 0, 2).tolist() == [-1, -1]
    # negative zero ties with positive zero, lower index wins
    z = np.array([0.0, -0.0, 0.0, -0.0])
    assert oracle.topk_select(z, 4, 2).tolist() == [0, 1]


# ---------------------------------------------------------------- attention
def test_attention_reduces_to_sdpa():
    """sink -> -inf, no RoPE, every entry selected: plain softmax attention."""
    rng = _rng(7)
    H, d, R = 3, 32, 11
    q = rng.standard_normal((H, d))
    rows = rng.standard_normal((R, d))
    scale = 1 / math.sqrt(d)
    got = oracle.attend(q, 5, rows, np.full(H, -np.inf), scale, 0, THETA)
    tq = torch.from_numpy(q)[None, :, None, :]           # [1, H, 1, d]
    tk = torch.from_numpy(rows)[None, None].expand(1, H, R, d)
    mask = torch.ones(1, H, 1, R, dtype=torch.bool)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tk, attn_mask=mask,
                                                           scale=scale)
    np.testing.assert_allclose(got, ref[0, :, 0].numpy(), rtol=0, atol=1e-12)


def test_single_key_closed_form():
    """One visible entry, no window, sink -> -inf: o = R(p_j - t) e_j."""
    rng = _rng(8)
    d, r = 32, 16
    e = rng.standard_normal(d)
    pj, t = 12, 40
    row = oracle.rope(e[None], pj, r, THETA)
    q = rng.standard_normal((2, d))
    got = oracle.attend(q, t, row, np.full(2, -np.inf), 0.1, r, THETA)
    i = np.arange(r // 2)
    zz = (e[16::2] + 1j * e[17::2]) * np.exp(1j * (pj - t) * THETA ** (-2.0 * i / r))
    for h in range(2):
        np.testing.assert_allclose(got[h, :16], e[:16], atol=1e-12)
        np.testing.assert_allclose(got[h, 16::2], zz.real, atol=1e-12)
        np.testing.assert_allclose(got[h, 17::2], zz.imag, atol=1e-12)


def test_sink_closed_form_and_weight_sum():
    """q = 0 makes every logit 0: each of n rows weighs 1/(e^sink + n)."""
    d, n = 16, 7
    rows = np.zeros((n, d))
    rows[:, :8] = 1.0  # value 1 in the un-rotated dims, 0 in the rope dims
    sink = np.array([-np.inf, 0.0, 1.5, -2.0])
    got = oracle.attend(np.zeros((4, d)), 9, rows, sink, 0.25, 8, THETA)
    for h in range(4):
        want = n / (math.exp(sink[h]) + n) if np.isfinite(sink[h]) else 1.0
        np.testing.assert_allclose(got[h, :8], want, rtol=0, atol=1e-14)
        np.testing.assert_allclose(got[h, 8:], 0.0, atol=1e-14)
    assert got[0, 0] == pytest.approx(1.0, abs=1e-15)  # weights sum to 1
    assert np.all(got[1:, 0] < 1.0)                     # finite sink: below 1
    # random logits: the weight sum (value rows of ones) stays below 1
    rng = _rng(9)
    got2 = oracle.attend(rng.standard_normal((4, d)), 9, rows, sink, 0.25, 8, THETA)
    assert got2[0, 0] == pytest.approx(1.0, abs=1e-14)
    assert np.all(got2[1:, 0] < 1.0)


def test_attention_matches_brute_force():
    rng = _rng(10)
    H, d, r = 2, 12, 4
    q = rng.standard_normal((H, d))
    rows = rng.standard_normal((6, d))
    sink = rng.standard_normal(H)
    got = oracle.attend(q, 17, rows, sink, 0.3, r, THETA)
    ref = brute.attend(q.tolist(), 17, rows.tolist(), sink.tolist(), 0.3, r, THETA)
    np.testing.assert_allclose(got, np.array(ref), rtol=0, atol=1e-12)


def _tiny_layer(seed, T=64, d=16, r=8, H=2, HI=2, dI=8, k=5, W=6, width=8, stride=4):
    rng = _rng(seed)
    return dict(
        x=rng.standard_normal((T, d)), g=rng.standard_normal((T, d)),
        q_idx=rng.integers(-3, 4, size=(T, HI, dI)).astype(np.float64),
        w=np.exp2(rng.integers(-1, 2, size=(T, HI))).astype(np.float64),
        k_idx=rng.integers(-3, 4, size=((T - width) // stride + 1, dI)).astype(np.float64),
        q=rng.standard_normal((T, H, d)), sink=rng.standard_normal(H),
        kw=dict(width=width, stride=stride, topk=k, window=W, rope_dim=r, theta=THETA,
                scale=1 / math.sqrt(d)))


def test_whole_layer_matches_brute_force():
    L = _tiny_layer(11)
    kw = L["kw"]
    kv_cmp, kv_raw, idx, out = oracle.csa_prefill_layer(
        L["x"], L["g"], L["q_idx"], L["w"], L["k_idx"], L["q"], L["sink"], **kw)
    b_cmp = brute.compress(L["x"].tolist(), L["g"].tolist(), kw["width"], kw["stride"],
                           kw["rope_dim"], THETA)
    np.testing.assert_allclose(kv_cmp, np.array(b_cmp), atol=1e-12)
    T = L["x"].shape[0]
    for t in range(T):
        sc = brute.scores(L["q_idx"][t].tolist(), L["w"][t].tolist(), L["k_idx"].tolist())
        vis = brute.visible(t, len(b_cmp), kw["width"], kw["stride"])
        sel = brute.topk(sc, len(vis), kw["topk"])
        assert idx[t].tolist() == sel
        raw = [brute._rot(list(L["x"][u]), u, kw["rope_dim"], THETA)
               for u in brute.window(t, kw["window"], 0, T)]
        rows = [b_cmp[j] for j in sel if j >= 0] + raw
        ref = brute.attend(L["q"][t].tolist(), t, rows, L["sink"].tolist(), kw["scale"],
                           kw["rope_dim"], THETA)
        np.testing.assert_allclose(out[t], np.array(ref), atol=1e-12)


def test_sparse_equals_dense_when_k_covers_all():
    L = _tiny_layer(12, k=100)
    kw = L["kw"]
    kv_cmp, kv_raw, idx, out = oracle.csa_prefill_layer(
        L["x"], L["g"], L["q_idx"], L["w"], L["k_idx"], L["q"], L["sink"], **kw)
    T = L["x"].shape[0]
    dense = oracle.hca_attn(L["q"], np.arange(T), kv_cmp, kv_cmp.shape[0], kv_raw, 0, T,
                            L["sink"], kw["scale"], kw["window"], kw["width"], kw["stride"],
                            kw["rope_dim"], THETA)
    np.testing.assert_allclose(out, dense, rtol=0, atol=1e-13)


def test_hca_is_csa_path_with_128_pooling():
    rng = _rng(13)
    T, d, H = 600, 16, 2
    x, g = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    q, sink = rng.standard_normal((T, H, d)), rng.standard_normal(H)
    kv = oracle.compress(x, g, 128, 128, 8, THETA)
    raw = oracle.rotate_raw(x, 0, 8, THETA)
    rows = np.array([0, 126, 127, 128, 300, 599])
    a = oracle.hca_attn(q, np.arange(T), kv, kv.shape[0], raw, 0, T, sink, 0.25, 128,
                        128, 128, 8, THETA, rows)
    all_idx = np.tile(np.arange(64), (T, 1))
    all_idx = np.where(all_idx < np.array([oracle.n_visible(t, kv.shape[0], 128, 128)
                                           for t in range(T)])[:, None], all_idx, -1)
    b = oracle.sparse_attn(q, np.arange(T), kv, all_idx, raw, 0, T, sink, 0.25, 128, 8,
                           THETA, rows)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_shift_of_all_positions_leaves_output_unchanged():
    L = _tiny_layer(14)
    kw = L["kw"]
    T = L["x"].shape[0]
    outs = []
    for shift in (0, 1000, 77777):
        kv_cmp = oracle.compress(L["x"], L["g"], kw["width"], kw["stride"], kw["rope_dim"],
                                 THETA, pos_offset=shift)
        kv_raw = oracle.rotate_raw(L["x"], shift, kw["rope_dim"], THETA)
        idx = oracle.index_topk(L["q_idx"], L["w"], L["k_idx"], np.arange(T), kv_cmp.shape[0],
                                kw["width"], kw["stride"], kw["topk"])
        res = []
        for t in range(T):
            rows = oracle.gather_rows(kv_cmp, idx[t], kv_raw, t, kw["window"], 0, T)
            res.append(oracle.attend(L["q"][t], t + shift, rows, L["sink"], kw["scale"],
                                     kw["rope_dim"], THETA))
        outs.append(np.stack(res))
    np.testing.assert_allclose(outs[1], outs[0], rtol=0, atol=1e-10)
    np.testing.assert_allclose(outs[2], outs[0], rtol=0, atol=1e-9)


# ---------------------------------------------------------------- decode-time append
@pytest.mark.parametrize("width,stride", [(8, 4), (128, 128), (2, 2), (5, 3)])
def test_append_equals_batch_compression_in_any_split(width, stride):
    # token arrivals cut at random points (single tokens, bursts, none): the
    # appended entries and raw rows, in order, are exactly the batch
    # compression and rotation of the whole sequence, each entry appearing
    # once, as soon as its last token has arrived
    rng = _rng(60 + width)
    T, d, r = 400, 16, 8
    x, g = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    full = oracle.compress(x, g, width, stride, r, THETA, pos_offset=3)
    full_raw = oracle.rotate_raw(x, 0, r, THETA)
    cuts = np.unique(np.concatenate([[0, T], rng.integers(0, T, 40), np.arange(0, 30)]))
    ents, raws, seen = [], [], 0
    for t_old, t_new in zip(cuts[:-1], cuts[1:]):
        # the window holds just the tokens from the first new entry's start
        # (or t_old), plus a few before
        j_first = oracle.n_compressed(int(t_old), width, stride)
        lo = max(0, min(stride * j_first, int(t_old)) - 3)
        j0, e, raw = oracle.compress_append(x[lo:t_new], g[lo:t_new], lo, int(t_old), int(t_new),
                                            width, stride, r, THETA, pos_offset=3)
        assert j0 == seen
        for k in range(e.shape[0]):  # entry j exists once its last token has arrived
            assert stride * (j0 + k) + width - 1 < t_new
        seen += e.shape[0]
        ents.append(e)
        raws.append(raw)
    assert seen == full.shape[0] == oracle.n_compressed(T, width, stride)
    np.testing.assert_array_equal(np.concatenate(ents), full)
    np.testing.assert_array_equal(np.concatenate(raws), full_raw)


def test_append_of_one_token_against_brute_force():
    # the token that completes entry j = 5 (tokens 20..27 at stride 4)
    # creates exactly that entry, equal to the brute-force pooling of those
    # taps rotated at position 20
    rng = _rng(64)
    x, g = rng.standard_normal((28, 8)), rng.standard_normal((28, 8))
    j0, e, raw = oracle.compress_append(x[18:], g[18:], 18, 27, 28, 8, 4, 4, THETA)
    assert j0 == 5 and e.shape[0] == 1
    ref = brute.compress(x[20:28].tolist(), g[20:28].tolist(), 8, 4, 4, THETA, pos_offset=20)
    np.testing.assert_allclose(e[0], np.array(ref[0]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(raw[0], np.array(brute._rot(list(x[27]), 27, 4, THETA)),
                               rtol=0, atol=1e-12)
    # the tokens before it complete nothing new; a window that lacks a tap fails
    j0, e, _ = oracle.compress_append(x[18:], g[18:], 18, 25, 27, 8, 4, 4, THETA)
    assert (j0, e.shape[0]) == (5, 0)
    with pytest.raises(ValueError):
        oracle.compress_append(x[21:], g[21:], 21, 27, 28, 8, 4, 4, THETA)


# ---------------------------------------------------------------- HCA prefill
def test_hca_prefill_layer_matches_brute_force():
    # every token attends to all entries whose 128 tokens it has seen, plus
    # its window, with the sink; pooling 128 -> 1 without overlap
    rng = _rng(65)
    T, d, H, r, W = 300, 8, 2, 4, 16
    x, g = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    q, sink = rng.standard_normal((T, H, d)), rng.standard_normal(H)
    rows = np.array([0, 126, 127, 128, 255, 256, 299])
    kv_cmp, kv_raw, out = oracle.hca_prefill_layer(x, g, q, sink, window=W, rope_dim=r,
                                                   theta=THETA, scale=0.3, rows=rows)
    assert kv_cmp.shape[0] == 2
    b_cmp = brute.compress(x.tolist(), g.tolist(), 128, 128, r, THETA)
    np.testing.assert_allclose(kv_cmp, np.array(b_cmp), rtol=0, atol=1e-12)
    for i, t in enumerate(rows):
        vis = [b_cmp[j] for j in brute.visible(int(t), len(b_cmp), 128, 128)]
        raw = [brute._rot(list(x[u]), u, r, THETA) for u in brute.window(int(t), W, 0, T)]
        ref = brute.attend(q[t].tolist(), int(t), vis + raw, sink.tolist(), 0.3, r, THETA)
        np.testing.assert_allclose(out[i], np.array(ref), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    """A wrong rotation sign or a dropped sink term in the oracle must trip a pin."""
    good_rope = csa_oracle.rope

    def bad_rope(x, pos, rope_dim, theta):
        return good_rope(x, -np.asarray(pos), rope_dim, theta)

    monkeypatch.setattr(csa_oracle, "rope", bad_rope)
    monkeypatch.setattr(oracle, "rope", bad_rope)
    with pytest.raises(AssertionError):
        test_rope_is_complex_rotation()
    with pytest.raises(AssertionError):
        test_single_key_closed_form()
    monkeypatch.setattr(csa_oracle, "rope", good_rope)
    monkeypatch.setattr(oracle, "rope", good_rope)

    good_attend = csa_oracle.attend

    def no_sink(q, t, rows, sink, scale, rope_dim, theta):
        return good_attend(q, t, rows, np.full_like(np.asarray(sink, float), -np.inf), scale,
                           rope_dim, theta)

    monkeypatch.setattr(csa_oracle, "attend", no_sink)
    monkeypatch.setattr(oracle, "attend", no_sink)
    with pytest.raises(AssertionError):
        test_sink_closed_form_and_weight_sum()
    monkeypatch.setattr(csa_oracle, "attend", good_attend)
    monkeypatch.setattr(oracle, "attend", good_attend)


def test_pins_catch_half_split_rope(monkeypatch):
    """RoPE pairs (r0 + i, r0 + i + r/2) instead of the interleaved pairs
    (r0 + 2i, r0 + 2i + 1) must trip the brute-force and closed-form pins."""
    good_rope = csa_oracle.rope

    def half_split(x, pos, rope_dim, theta):
        x = np.asarray(x, dtype=np.float64)
        r0, h = x.shape[-1] - rope_dim, rope_dim // 2
        perm = r0 + np.stack([np.arange(h), np.arange(h) + h], axis=1).reshape(-1)
        y = x.copy()
        y[..., r0:] = x[..., perm]   # half-split pairs moved to interleaved slots
        z = good_rope(y, pos, rope_dim, theta)
        out = z.copy()
        out[..., perm] = z[..., r0:]
        return out

    monkeypatch.setattr(csa_oracle, "rope", half_split)
    monkeypatch.setattr(oracle, "rope", half_split)
    with pytest.raises(AssertionError):
        test_rope_is_complex_rotation()
    with pytest.raises(AssertionError):
        test_whole_layer_matches_brute_force()


def test_pins_catch_transposed_score_matrix(monkeypatch):
    """Attention weights normalised over the heads instead of over the rows
    (the query-by-row score matrix used transposed) must trip the SDPA
    reduction and the brute-force pin."""

    def transposed(q, t, rows, sink, scale, rope_dim, theta):
        qh = csa_oracle.rope(q, t, rope_dim, theta)
        rows = np.asarray(rows, dtype=np.float64)
        z = (rows @ qh.T) * scale * csa_oracle.attention_temperature(theta)  # [R, H]
        z = np.concatenate([z, np.asarray(sink, dtype=np.float64)[None, :]], axis=0)
        with np.errstate(invalid="ignore"):  # a sink of -inf: its own row is NaN, dropped
            e = np.exp(z - z.max(axis=1, keepdims=True))
        a = (e / e.sum(axis=1, keepdims=True))[:-1]  # rows of a softmax over the heads
        return csa_oracle.rope(a.T @ rows, -t, rope_dim, theta)

    monkeypatch.setattr(csa_oracle, "attend", transposed)
    monkeypatch.setattr(oracle, "attend", transposed)
    with pytest.raises(AssertionError):
        test_attention_reduces_to_sdpa()
    with pytest.raises(AssertionError):
        test_attention_matches_brute_force()


# ---------------------------------------------------------------- YaRN
# The compressed layers' extended RoPE ("Partial RoPE" rows: theta = 160,000
# with YaRN, factor 16 over 65,536 tokens), pinned to what the published
# definition fixes (Peng et al. 2023, section 3) without retyping it: the
# end points of the ramp, its bounds, the temperature's closed form, the
# rotation's relative-distance property and the pure-Python brute force.
V4_YARN = oracle.YaRN(theta=160000.0, factor=16.0, orig_ctx=65536)
V4_YARN_TUPLE = (160000.0, 16.0, 65536, 32.0, 1.0)


def test_yarn_with_factor_one_is_plain_rope():
    x = _rng(40).standard_normal((5, 32))
    pos = np.array([0, 3, 70000, 1 << 20, -9])
    plain = oracle.rope(x, pos, 16, 160000.0)
    spec = oracle.YaRN(theta=160000.0, factor=1.0, orig_ctx=65536)
    np.testing.assert_array_equal(oracle.rope(x, pos, 16, spec), plain)
    assert oracle.attention_temperature(spec) == 1.0


def test_yarn_keeps_the_fastest_pair_and_slows_the_slowest_by_the_factor():
    f = oracle.rope_freqs(64, V4_YARN)
    base = 160000.0 ** (-np.arange(32) * 2.0 / 64)
    # pair 0 turns once per token: 65,536 / (2 pi) >> 32 turns over the context
    assert f[0] == 1.0
    # pair 31 turns 0.1 times over 65,536 tokens (< 1): interpolated by 16
    assert 65536 * base[31] / (2 * math.pi) < 1.0
    assert f[31] == base[31] / 16.0
    # every pair lies between its interpolated and original frequency, and
    # the interpolation never speeds a pair up
    assert np.all(f <= base * (1 + 1e-15)) and np.all(f >= base / 16.0 * (1 - 1e-15))
    assert np.all(np.diff(f / base) <= 1e-15)  # slower pairs are interpolated more


def test_yarn_temperature_closed_form_and_one_key_attention():
    tau = oracle.attention_temperature(V4_YARN)
    assert tau == pytest.approx((1 + 0.1 * math.log(16.0)) ** 2, rel=1e-15)
    assert tau == pytest.approx(1.63139, abs=1e-5)
    # one key e at position p, no rope dims rotated for the dot product
    # check: with rope_dim 0, a = exp(tau s z) / (exp(sink) + exp(tau s z))
    rng = _rng(41)
    q, e, sink = rng.standard_normal((3, 8)), rng.standard_normal((1, 8)), rng.standard_normal(3)
    out = oracle.attend(q, 50, e, sink, 0.25, 0, V4_YARN)
    z = tau * 0.25 * (q @ e[0])
    a = np.exp(z) / (np.exp(sink) + np.exp(z))
    np.testing.assert_allclose(out, a[:, None] * e, rtol=0, atol=1e-14)


def test_yarn_rotation_depends_only_on_relative_distance():
    rng = _rng(42)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for a, b, shift in ((10, 3, 1000), (70000, 5, 123456), (0, 300000, 77)):
        d0 = oracle.rope(q, a, 64, V4_YARN) @ oracle.rope(k, b, 64, V4_YARN)
        d1 = oracle.rope(q, a + shift, 64, V4_YARN) @ oracle.rope(k, b + shift, 64, V4_YARN)
        assert d0 == pytest.approx(d1, rel=1e-9, abs=1e-9)
    back = oracle.rope(oracle.rope(q, 98765, 64, V4_YARN), -98765, 64, V4_YARN)
    np.testing.assert_allclose(back, q, atol=1e-12)


def test_yarn_layer_matches_brute_force():
    # a tiny layer whose positions run past the original context (L = 40)
    L = _tiny_layer(43, T=96)
    kw = dict(L["kw"])
    # rope_dim 8, base 500, L 40: pair 0 turns 6.4 times over L (kept, above
    # beta = 4), pair 1 1.3 times (on the ramp), pairs 2-3 under once (slowed)
    spec = oracle.YaRN(theta=500.0, factor=4.0, orig_ctx=40, beta_fast=4.0, beta_slow=1.0)
    tup = (500.0, 4.0, 40, 4.0, 1.0)
    kw["theta"] = spec
    kv_cmp, kv_raw, idx, out = oracle.csa_prefill_layer(
        L["x"], L["g"], L["q_idx"], L["w"], L["k_idx"], L["q"], L["sink"], **kw)
    b_cmp = brute.compress(L["x"].tolist(), L["g"].tolist(), kw["width"], kw["stride"],
                           kw["rope_dim"], tup)
    np.testing.assert_allclose(kv_cmp, np.array(b_cmp), atol=1e-12)
    T = L["x"].shape[0]
    for t in (0, 7, 40, 95):
        sel = [j for j in idx[t].tolist() if j >= 0]
        raw = [brute._rot(list(L["x"][u]), u, kw["rope_dim"], tup)
               for u in brute.window(t, kw["window"], 0, T)]
        rows = [b_cmp[j] for j in sel] + raw
        ref = brute.attend(L["q"][t].tolist(), t, rows, L["sink"].tolist(), kw["scale"],
                           kw["rope_dim"], tup)
        np.testing.assert_allclose(out[t], np.array(ref), atol=1e-12)
    # the ramp of this spec is exercised: some pairs interpolated, some kept
    f = oracle.rope_freqs(kw["rope_dim"], spec)
    plain = oracle.rope_freqs(kw["rope_dim"], 500.0)
    assert f[0] == plain[0] and plain[1] / 4 < f[1] < plain[1]
    np.testing.assert_array_equal(f[2:], plain[2:] / 4)


# ---------------------------------------------------------------- CSA2
def test_csa2_full_and_reuse_layers_match_brute_force():
    # "CSA2 encoder layers (2x compression, Full + Reuse)": KV pooled 2 -> 1
    # and computed in a Full layer; a Reuse layer attends with its own
    # queries over the Full layer's entries and top-k selection
    L = _tiny_layer(44, T=40, width=2, stride=2, k=6)
    kw = L["kw"]
    T = L["x"].shape[0]
    kv_cmp, kv_raw, idx, out = oracle.csa_prefill_layer(
        L["x"], L["g"], L["q_idx"], L["w"],
        _rng(45).integers(-3, 4, size=(T // 2, L["q_idx"].shape[2])).astype(np.float64),
        L["q"], L["sink"], **kw)
    assert kv_cmp.shape[0] == T // 2  # non-overlapping pairs: floor(T / 2) entries
    b_cmp = brute.compress(L["x"].tolist(), L["g"].tolist(), 2, 2, kw["rope_dim"], THETA)
    np.testing.assert_allclose(kv_cmp, np.array(b_cmp), atol=1e-12)
    q2 = _rng(46).standard_normal(L["q"].shape)
    sink2 = _rng(47).standard_normal(L["sink"].shape)
    reuse = oracle.sparse_attn(q2, np.arange(T), kv_cmp, idx, kv_raw, 0, T, sink2, kw["scale"],
                               kw["window"], kw["rope_dim"], THETA)
    for t in (0, 1, 2, 17, 39):
        sel = [j for j in idx[t].tolist() if j >= 0]
        assert all(2 * j + 1 <= t for j in sel)  # a pair is visible once both tokens are
        raw = [brute._rot(list(L["x"][u]), u, kw["rope_dim"], THETA)
               for u in brute.window(t, kw["window"], 0, T)]
        rows = [b_cmp[j] for j in sel] + raw
        ref = brute.attend(q2[t].tolist(), t, rows, sink2.tolist(), kw["scale"], kw["rope_dim"],
                           THETA)
        np.testing.assert_allclose(reuse[t], np.array(ref), atol=1e-12)


# ---------------------------------------------------------------- FP8 KV cache
# The cache quantized after RoPE ("Partial RoPE" row of "DeepSeek-V4.1-Flash
# vs Inkling"), read as OCP E4M3 with one fp32 scale per row: pinned to the
# format's stated points, to torch's float8_e4m3fn conversion (a library
# routine, round to nearest even) and to the rounding error bound.
def test_e4m3_code_table_has_the_format_points():
    v = oracle.e4m3_values()
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0          # largest finite
    assert v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9   # smallest normal, subnormal
    assert v[0x38] == 1.0 and v[0x00] == 0.0 and np.signbit(v[0x80])
    assert [c for c in range(256) if np.isnan(v[c])] == [0x7F, 0xFF]
    assert np.all(np.diff(v[:127]) > 0)                     # codes 0..126 increase
    np.testing.assert_array_equal(v[128:255], -v[:127])     # sign bit


def test_e4m3_encode_matches_torch_float8_e4m3fn():
    rng = _rng(80)
    v = oracle.e4m3_values()[:127]
    mids = (v[1:] + v[:-1]) / 2                              # every tie between neighbours
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 1e-2,
                        rng.standard_normal(5000) * 2 ** -8, mids, -mids, v, -v]).astype(np.float32)
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_quantized_rows_round_trip_and_error_bound():
    rng = _rng(81)
    rows = (rng.standard_normal((40, 512)) * np.exp(rng.uniform(-6, 6, (40, 1)))).astype(np.float32)
    rows[3] = 0.0
    codes, scales = oracle.quantize_fp8_rows(rows)
    back = oracle.dequantize_fp8_rows(codes, scales)
    assert scales[3] == 1.0 and np.all(codes[3] == 0)       # an all-zero row
    for r in range(40):
        j = int(np.argmax(np.abs(rows[r])))
        if rows[r, j] != 0:                                   # the largest maps to +-448
            assert abs(oracle.e4m3_values()[codes[r, j]]) == 448.0
    # relative half-step of 3 mantissa bits for normals, absolute half of the
    # smallest subnormal step below 2^-6 (both in units of the row's scale)
    y = np.abs(rows / scales[:, None].astype(np.float64))
    bound = np.where(y >= 2.0 ** -6, y * 2.0 ** -4, 2.0 ** -10) * scales[:, None] * (1 + 1e-6)
    assert np.all(np.abs(back - rows) <= bound)
    # rows made of code values times a power-of-two scale come back exactly
    exact = oracle.e4m3_values()[rng.integers(0, 127, (5, 64))] * 2.0 ** -3
    exact[:, 0] = 448 * 2.0 ** -3
    c2, s2 = oracle.quantize_fp8_rows(exact)
    np.testing.assert_array_equal(oracle.dequantize_fp8_rows(c2, s2), exact)
