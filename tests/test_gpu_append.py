"""Decode-time compression through the C ABI (csa_compress_append): the
entries and rotated raw rows that newly arrived tokens complete, against the
oracle's compress_append, against the whole-sequence call on the GPU, and
the device-side range check."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev, host64
from sparse_compressed_attention_csa_b200 import CsaError, Params, csa_poll_device_error, layer
from sparse_compressed_attention_csa_b200 import csa_compress
from sparse_compressed_attention_csa_b200.workloads import bf16_bits, bits_to_f32

pytestmark = pytest.mark.gpu

D, R, THETA = 512, 64, 10000.0
SENTINEL = 0x7F7F  # a bf16 pattern no written row produces here


def _i32(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


def _bf16_rows(rng, shape):
    return bf16_bits(rng.standard_normal(shape).astype(np.float32))


def test_append_matches_oracle_and_leaves_other_rows():
    # three sequences: 4 tokens completing entry 249 (tokens 996..1003),
    # 33 tokens from position 7 (entries 0..8), 17 tokens (entries 129..133)
    width, stride = 8, 4
    p = Params(d=D, rope_dim=R, theta=THETA, width=width, stride=stride)
    t_old, t_new, x_pos0 = [1000, 7, 523], [1004, 40, 540], [990, 0, 510]
    B, L, n_cap, raw_cap = 3, 64, 300, 1100
    rng = np.random.default_rng(70)
    x, g = _bf16_rows(rng, (B, L, D)), _bf16_rows(rng, (B, L, D))
    kv_cmp = torch.full((B, n_cap, D), SENTINEL, dtype=torch.int16, device="cuda")
    kv_raw = torch.full((B, raw_cap, D), SENTINEL, dtype=torch.int16, device="cuda")
    layer.append_tokens(p, dev(x), dev(g), _i32(x_pos0), _i32(t_old), _i32(t_new), 33,
                        kv_cmp.view(torch.bfloat16), kv_raw.view(torch.bfloat16),
                        _i32([0, 0, 0]))
    csa_poll_device_error()
    got_c, got_r = kv_cmp.cpu().numpy().view(np.uint16), kv_raw.cpu().numpy().view(np.uint16)
    for b in range(B):
        j0, ent, raw = oracle.compress_append(bits_to_f32(x[b]), bits_to_f32(g[b]), x_pos0[b],
                                              t_old[b], t_new[b], width, stride, R, THETA)
        j1 = j0 + ent.shape[0]
        assert ent.shape[0] == [1, 9, 5][b]
        assert_close(bits_to_f32(got_c[b, j0:j1]).astype(np.float64), ent, "bf16", "entries")
        assert_close(bits_to_f32(got_r[b, t_old[b]:t_new[b]]).astype(np.float64), raw, "bf16",
                     "raw rows")
        keep_c = np.ones(n_cap, bool)
        keep_c[j0:j1] = False
        keep_r = np.ones(raw_cap, bool)
        keep_r[t_old[b]:t_new[b]] = False
        assert np.all(got_c[b][keep_c] == SENTINEL) and np.all(got_r[b][keep_r] == SENTINEL)


@pytest.mark.parametrize("width,stride,dtype", [(8, 4, "bf16"), (128, 128, "bf16"),
                                                (2, 2, "bf16"), (8, 4, "f32")])
def test_append_token_stream_equals_whole_sequence(width, stride, dtype):
    # tokens arrive in bursts of 0..6 (ragged across the two sequences); the
    # caches built by appending equal, bit for bit, what the whole-sequence
    # call writes, and match the oracle
    T, B = 700, 2
    p = Params(d=D, rope_dim=R, theta=THETA, width=width, stride=stride)
    rng = np.random.default_rng(71 + width)
    xf = rng.standard_normal((B, T, D)).astype(np.float32)
    gf = rng.standard_normal((B, T, D)).astype(np.float32)
    if dtype == "bf16":
        x, g = dev(bf16_bits(xf)), dev(bf16_bits(gf))
    else:
        x, g = dev(xf), dev(gf)
    N = (T - width) // stride + 1
    whole_c = torch.empty((B, N, D), dtype=x.dtype, device="cuda")
    whole_r = torch.empty((B, T, D), dtype=x.dtype, device="cuda")
    csa_compress(p, x, g, whole_c, whole_r)
    app_c = torch.zeros_like(whole_c)
    app_r = torch.zeros_like(whole_r)
    zeros = _i32([0] * B)
    t = np.zeros(B, dtype=np.int64)
    while np.any(t < T):
        step = np.minimum(rng.integers(0, 7, size=B), T - t)
        layer.append_tokens(p, x, g, zeros, _i32(t.tolist()), _i32((t + step).tolist()), 6,
                            app_c, app_r, zeros)
        t += step
    csa_poll_device_error()
    assert torch.equal(app_c, whole_c) and torch.equal(app_r, whole_r)
    xs = bits_to_f32(bf16_bits(xf)) if dtype == "bf16" else xf
    gs = bits_to_f32(bf16_bits(gf)) if dtype == "bf16" else gf
    for b in range(B):
        want = oracle.compress(xs[b].astype(np.float64), gs[b].astype(np.float64), width, stride,
                               R, THETA)
        assert_close(host64(app_c[b]), want, dtype, "appended entries")


def test_append_range_breaking_the_rules_is_reported():
    # more new tokens than max_new: the sequence is skipped whole; entries
    # past the cache: those rows are skipped; both record
    # CSA_ERR_DEVICE_BOUNDS (status 8)
    p = Params(d=D, rope_dim=R, theta=THETA, width=8, stride=4)
    rng = np.random.default_rng(72)
    x, g = dev(_bf16_rows(rng, (1, 64, D))), dev(_bf16_rows(rng, (1, 64, D)))
    kv = torch.full((1, 4, D), SENTINEL, dtype=torch.int16, device="cuda")
    written = []
    for max_new in (8, 40):  # 40 tokens > 8; then entries 4..8 >= n_cap 4
        csa_poll_device_error()
        layer.append_tokens(p, x, g, _i32([0]), _i32([0]), _i32([40]), max_new,
                            kv.view(torch.bfloat16))
        with pytest.raises(CsaError) as ei:
            csa_poll_device_error()
        assert ei.value.status == 8
        written.append(kv.cpu().numpy().view(np.uint16) != SENTINEL)
    csa_poll_device_error()
    assert not np.any(written[0])  # skipped whole
    assert np.all(written[1])      # entries 0..3, the ones that fit
