"""Property-based pins of the oracle: small shapes and values drawn at
random (hypothesis), checked against the independent pure-Python brute
force (tests/brute.py) and against properties the mathematics fixes.

Ties, signed zeros, empty and ragged sizes come up far more often here than
in the fixed-seed pins; each property holds for every draw, and the example
counts keep the file to a few seconds on the CPU.
"""
import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import brute
import oracle

SETTINGS = settings(max_examples=60, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])
THETA = 10000.0

# values with many ties, both zeros and negatives
_TIED = st.sampled_from([-2.0, -1.0, -0.0, 0.0, 0.5, 1.0, 2.5])


@SETTINGS
@given(vals=st.lists(_TIED, min_size=1, max_size=60), data=st.data())
def test_topk_select_equals_sorting_by_score_then_index(vals, data):
    # "keeps the top 1,024 entries": the k largest, ties to the lower index,
    # -0.0 tied with +0.0, ascending indices, -1 padding past the visible ones
    n = len(vals)
    n_vis = data.draw(st.integers(0, n))
    k = data.draw(st.integers(1, n + 8))
    got = oracle.topk_select(np.array(vals, dtype=np.float64), n_vis, k)
    assert got.tolist() == brute.topk(vals, n_vis, k)


@SETTINGS
@given(ws=st.sampled_from([(8, 4), (4, 4), (2, 2), (3, 1), (5, 2), (6, 6)]),
       T=st.integers(0, 22), d=st.sampled_from([2, 4, 6]), rope=st.sampled_from([0, 2, "all"]),
       pos_offset=st.sampled_from([0, 3]), seed=st.integers(0, 2 ** 31))
def test_compress_equals_brute_force(ws, T, d, rope, pos_offset, seed):
    width, stride = ws
    rope_dim = d if rope == "all" else rope
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    g = 2.0 * rng.standard_normal((T, d))
    got = oracle.compress(x, g, width, stride, rope_dim, THETA, pos_offset)
    want = (np.array(brute.compress(x.tolist(), g.tolist(), width, stride, rope_dim, THETA,
                                    pos_offset)).reshape(-1, d)
            if T else np.zeros((0, d)))  # no tokens, no entries
    assert got.shape == want.shape == (oracle.n_compressed(T, width, stride), d)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@SETTINGS
@given(H=st.integers(1, 3), d=st.sampled_from([2, 4]), R=st.integers(1, 6),
       t=st.integers(0, 5000), rope_dim=st.sampled_from([0, 2]), seed=st.integers(0, 2 ** 31))
def test_attend_equals_brute_force(H, d, R, t, rope_dim, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((H, d))
    rows = rng.standard_normal((R, d))
    sink = rng.standard_normal(H)
    scale = 1.0 / math.sqrt(d)
    got = oracle.attend(q, t, rows, sink, scale, rope_dim, THETA)
    want = np.array(brute.attend(q.tolist(), t, rows.tolist(), sink.tolist(), scale, rope_dim,
                                 THETA))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@SETTINGS
@given(a=st.integers(-70000, 70000), b=st.integers(-70000, 70000),
       rope_dim=st.sampled_from([2, 4, 8]), seed=st.integers(0, 2 ** 31))
def test_rope_rotations_compose(a, b, rope_dim, seed):
    # rotating by a then by b is rotating by a + b (each pair turns at its
    # own fixed frequency), and the non-rotated dims never change
    x = np.random.default_rng(seed).standard_normal(rope_dim + 3)
    ab = oracle.rope(oracle.rope(x, a, rope_dim, THETA), b, rope_dim, THETA)
    np.testing.assert_allclose(ab, oracle.rope(x, a + b, rope_dim, THETA), rtol=0, atol=1e-9)
    assert np.array_equal(ab[:3], x[:3])
    np.testing.assert_allclose(np.linalg.norm(ab), np.linalg.norm(x), rtol=1e-12)


@SETTINGS
@given(t=st.integers(0, 3000), n_cmp=st.integers(0, 800),
       ws=st.sampled_from([(8, 4), (2, 2), (128, 128), (5, 3)]))
def test_visible_entry_count_equals_enumeration(t, n_cmp, ws):
    width, stride = ws
    assert oracle.n_visible(t, n_cmp, width, stride) == len(brute.visible(t, n_cmp, width,
                                                                          stride))


@SETTINGS
@given(t=st.integers(0, 400), W=st.integers(1, 160), raw_pos0=st.integers(0, 400),
       n_raw=st.integers(0, 200))
def test_window_tokens_equal_enumeration(t, W, raw_pos0, n_raw):
    assert oracle.window_tokens(t, W, raw_pos0, n_raw).tolist() == brute.window(t, W, raw_pos0,
                                                                                n_raw)


@SETTINGS
@given(n=st.integers(1, 6), d=st.sampled_from([1, 8, 33]), log_mag=st.floats(-12, 12),
       zero_row=st.booleans(), seed=st.integers(0, 2 ** 31))
def test_fp8_rows_decode_within_half_a_code_step(n, d, log_mag, zero_row, seed):
    # E4M3 has 3 mantissa bits: a normal value decodes within 2^-4 of itself
    # (relative); below 2^-6 (subnormal) within half the 2^-9 step; the
    # row's largest magnitude lands on 448 (the largest finite code)
    rng = np.random.default_rng(seed)
    rows = (rng.standard_normal((n, d)) * 10.0 ** log_mag).astype(np.float32)
    if zero_row:
        rows[0] = 0.0
    codes, scales = oracle.quantize_fp8_rows(rows)
    assert codes.dtype == np.uint8 and not np.any((codes & 0x7F) == 0x7F)  # no NaN code
    back = oracle.dequantize_fp8_rows(codes, scales)
    y = rows.astype(np.float64) / scales.astype(np.float64)[:, None]
    err = np.abs(back / scales.astype(np.float64)[:, None] - y)
    bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    amax = np.abs(rows).max(axis=1)
    for r in range(n):
        if amax[r] > 0:
            assert np.abs(back[r]).max() == 448.0 * float(scales[r])
        else:
            assert scales[r] == 1.0 and np.all(back[r] == 0.0)


@SETTINGS
@given(H=st.integers(1, 4), dI=st.integers(1, 8), N=st.integers(0, 20),
       seed=st.integers(0, 2 ** 31))
def test_index_scores_integer_inputs_exact(H, dI, N, seed):
    # integer keys and queries with power-of-two weights: every score is an
    # exact binary value, so the oracle and the brute force agree bit for bit
    rng = np.random.default_rng(seed)
    q = rng.integers(-8, 9, (H, dI)).astype(np.float64)
    w = 2.0 ** rng.integers(-2, 3, H)
    k = rng.integers(-8, 9, (N, dI)).astype(np.float64)
    got = oracle.index_scores(q[None], w[None], k)[0]
    assert got.tolist() == brute.scores(q.tolist(), w.tolist(), k.tolist())


_YARN = st.builds(oracle.YaRN, theta=st.sampled_from([10000.0, 160000.0, 500.0]),
                  factor=st.sampled_from([1.0, 4.0, 16.0]),
                  orig_ctx=st.sampled_from([40, 4096, 65536]))


@SETTINGS
@given(spec=_YARN, rope_dim=st.sampled_from([4, 16, 64]))
def test_yarn_frequencies_lie_between_the_scaled_and_the_original(spec, rope_dim):
    # each pair's frequency is a blend of f / s and f with a weight in
    # [0, 1]: it lies between the two, and it falls with the pair index
    f = oracle.rope_freqs(rope_dim, spec.theta)
    fy = oracle.rope_freqs(rope_dim, spec)
    assert np.all(fy <= f * (1 + 1e-15)) and np.all(fy >= f / spec.factor * (1 - 1e-15))
    assert np.all(np.diff(fy) < 0)


@SETTINGS
@given(spec=_YARN, a=st.integers(-200000, 200000), b=st.integers(-200000, 200000),
       seed=st.integers(0, 2 ** 31))
def test_yarn_rotations_compose(spec, a, b, seed):
    x = np.random.default_rng(seed).standard_normal(8 + 2)
    ab = oracle.rope(oracle.rope(x, a, 8, spec), b, 8, spec)
    np.testing.assert_allclose(ab, oracle.rope(x, a + b, 8, spec), rtol=0, atol=1e-9)
    assert np.array_equal(ab[:2], x[:2])


@SETTINGS
@given(ws=st.sampled_from([(8, 4), (2, 2), (5, 3), (16, 16), (4, 1)]), T=st.integers(0, 120),
       cuts=st.lists(st.integers(0, 120), max_size=12), back=st.integers(0, 5),
       seed=st.integers(0, 2 ** 31))
def test_append_at_any_cuts_equals_whole_sequence(ws, T, cuts, back, seed):
    # tokens arrive in bursts cut anywhere (empty bursts too), each burst
    # handed a window that starts at most `back` tokens before what it needs:
    # the appended entries and raw rows, in order, are the whole sequence's
    width, stride = ws
    rng = np.random.default_rng(seed)
    d, r = 4, 2
    x, g = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    bounds = sorted({0, T, *[c for c in cuts if c <= T]})
    ents, raws, seen = [], [], 0
    for t_old, t_new in zip(bounds[:-1], bounds[1:]):
        j_first = oracle.n_compressed(t_old, width, stride)
        lo = max(0, min(stride * j_first, t_old) - back)
        j0, e, raw = oracle.compress_append(x[lo:t_new], g[lo:t_new], lo, t_old, t_new, width,
                                            stride, r, THETA)
        assert j0 == seen
        seen += e.shape[0]
        ents.append(e)
        raws.append(raw)
    full = oracle.compress(x, g, width, stride, r, THETA)
    assert seen == full.shape[0]
    np.testing.assert_array_equal(np.concatenate(ents) if ents else np.zeros((0, d)), full)
    np.testing.assert_array_equal(np.concatenate(raws) if raws else np.zeros((0, d)),
                                  oracle.rotate_raw(x, 0, r, THETA))
