"""The seeded input recipe (CPU): reproducible draws, one stream per tensor,
and the value distributions the parity tests rely on (integer-valued
indexer inputs with power-of-two weights make every score exact)."""
import numpy as np

from sparse_compressed_attention_csa_b200 import workloads as W

SMALL_DECODE = W.CSA_DECODE_64K.replace(B=2, T=4 * 700 + 8, seed=5)
SMALL_PREFILL = W.CSA_PREFILL_8K.replace(T=300, seed=6)


def _same(a, b):
    assert a.keys() == b.keys()
    for k in a:
        assert a[k].dtype == b[k].dtype and np.array_equal(a[k], b[k]), k


def test_same_seed_same_inputs_other_seed_other_inputs():
    _same(W.generate(SMALL_DECODE), W.generate(SMALL_DECODE))
    other = W.generate(SMALL_DECODE.replace(seed=7))
    assert not np.array_equal(other["q"], W.generate(SMALL_DECODE)["q"])


def test_each_tensor_has_its_own_stream():
    full = W.generate(SMALL_DECODE)
    for keys in ({"q"}, {"k_idx", "kv_cmp"}, {"kv_raw"}):
        part = W.generate(SMALL_DECODE, keys=keys)
        for k in keys:
            assert np.array_equal(part[k], full[k]), k
    full_p = W.generate(SMALL_PREFILL)
    assert np.array_equal(W.generate(SMALL_PREFILL, keys={"g"})["g"], full_p["g"])


def test_value_recipe_bf16():
    d = W.generate(SMALL_DECODE)
    for k in ("q_idx", "k_idx"):
        v = W.to_f64(d[k])
        assert np.array_equal(v, np.round(v)) and v.min() >= -8 and v.max() <= 8, k
        assert set(np.unique(v)) == set(range(-8, 9)), k  # every integer of the range occurs
    assert set(np.unique(d["w"]).tolist()) <= {0.25, 0.5, 1.0, 2.0, 4.0}
    for k in ("q", "kv_cmp", "kv_raw"):
        v = W.to_f64(d[k])
        assert d[k].dtype == np.uint16 and np.all(np.isfinite(v)), k
        assert abs(v.mean()) < 0.05 and abs(v.std() - 1.0) < 0.05, k
    assert d["sink"].dtype == np.float32 and d["sink"].shape == (128,)


def test_value_recipe_tiny_f32():
    d = W.generate(W.TINY_F32)
    for k in ("q_idx", "k_idx"):
        v = d[k]
        assert v.dtype == np.float32 and np.array_equal(v, np.round(v))
        assert v.min() >= -3 and v.max() <= 3, k
    assert set(np.unique(d["w"]).tolist()) <= {0.5, 1.0, 2.0}


def test_positions_and_window_bookkeeping():
    d = W.generate(SMALL_DECODE)
    T, Wn = SMALL_DECODE.T, SMALL_DECODE.window
    assert np.all(d["q_pos"] == T - 1)                 # the last token queries
    assert np.all(d["raw_pos0"] == T - Wn) and np.all(d["n_raw"] == Wn)
    assert np.all(d["n_cmp"] == (T - 8) // 4 + 1)
    assert d["kv_cmp"].shape == (2, (T - 8) // 4 + 1, 512) and d["kv_raw"].shape == (2, Wn, 512)
    p = W.generate(SMALL_PREFILL)
    assert np.array_equal(p["q_pos"][0], np.arange(SMALL_PREFILL.T))
    assert "kv_cmp" not in p  # prefill pools its own entries on the path


def test_indexer_inputs_keep_every_fp32_sum_exact():
    # worst case over the recipe: a dot product of d_I integers of magnitude
    # <= r is at most d_I r^2; the score adds H_I of them times a weight of
    # at most 2^e_max; every value is a multiple of 2^e_min.  Below 2^24
    # units of 2^e_min, every partial sum in fp32 is exact, so the GPU's
    # scores (and the top-k decided on them) must equal the oracle's bit
    # for bit, whatever order the sums take
    for wl in (W.CSA_DECODE_64K, W.CSA_DECODE_1M, W.CSA_PREFILL_8K, W.TINY_F32, W.CSA2_DECODE):
        r = wl.int_range
        e_min, e_max = min(wl.w_exps), max(wl.w_exps)
        dot = wl.idx_dim * r * r
        assert dot < 2 ** 24, wl.name                       # the MMA's fp32 accumulation
        score_units = wl.idx_heads * dot * 2 ** (e_max - e_min)
        assert score_units < 2 ** 24, wl.name               # the weighted head sum
