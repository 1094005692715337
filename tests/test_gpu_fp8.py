"""FP8 KV cache (E4M3 codes with one fp32 scale per row, quantized after
RoPE) through the C ABI: the quantizer bit for bit against the oracle, and
the attention over quantized caches against the oracle's attention over the
caches its own quantization stands for."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev, host64, params_of, run_decode, theta_of
from sparse_compressed_attention_csa_b200 import (CSA_OP_HCA_ATTN, CSA_OP_SPARSE_ATTN,
                                                  csa_poll_device_error, csa_quantize_fp8,
                                                  csa_sparse_attn_fp8, csa_workspace_size,
                                                  hca_attn_fp8)
from sparse_compressed_attention_csa_b200 import workloads as W
from sparse_compressed_attention_csa_b200.workloads import bf16_bits, bits_to_f32, to_f64

pytestmark = pytest.mark.gpu


def _quantize(x_dev):
    codes = torch.empty(x_dev.shape, dtype=torch.uint8, device="cuda")
    scales = torch.empty(x_dev.shape[:-1], dtype=torch.float32, device="cuda")
    csa_quantize_fp8(x_dev, codes, scales)
    return codes, scales


def test_quantizer_matches_the_oracle_bit_for_bit():
    rng = np.random.default_rng(90)
    rows = (rng.standard_normal((300, 512)) * np.exp(rng.uniform(-20, 20, (300, 1))))
    rows[7] = 0.0
    rows[8, :] = 1e-5                                # E4M3 subnormal codes after scaling
    rows[8, 0] = 1.0
    rows[9, 5] = -1e30                               # one dominant element
    for dtype in ("bf16", "f32"):
        if dtype == "bf16":
            bits = bf16_bits(rows.astype(np.float32))
            x, vals = dev(bits), bits_to_f32(bits)
        else:
            vals = rows.astype(np.float32)
            x = dev(vals)
        codes, scales = _quantize(x)
        torch.cuda.synchronize()
        want_c, want_s = oracle.quantize_fp8_rows(vals)
        np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
        np.testing.assert_array_equal(codes.cpu().numpy(), want_c)


def _fp8_caches(data):
    """GPU and oracle views of the decode caches quantized after RoPE."""
    out = {}
    for key in ("kv_cmp", "kv_raw"):
        vals = bits_to_f32(data[key])
        codes, scales = _quantize(dev(data[key]))
        c_o, s_o = oracle.quantize_fp8_rows(vals)
        out[key] = (codes, scales, oracle.dequantize_fp8_rows(c_o, s_o))
    return out


def _check_csa_fp8(wl):
    data = W.generate(wl)
    p = params_of(wl)
    idx, _ = run_decode(wl, data)        # the indexer and top-k, as in the bf16 path
    q8 = _fp8_caches(data)
    t = {k: dev(data[k]) for k in ("q", "q_pos", "raw_pos0", "n_raw", "sink")}
    out = torch.empty_like(t["q"])
    nb = csa_workspace_size(p, CSA_OP_SPARSE_ATTN, wl.B, 1, wl.n_cmp)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    csa_sparse_attn_fp8(p, t["q"], t["q_pos"], q8["kv_cmp"][0], q8["kv_cmp"][1], idx,
                        q8["kv_raw"][0], q8["kv_raw"][1], t["raw_pos0"], t["n_raw"], t["sink"], out,
                        ws)
    torch.cuda.synchronize()
    csa_poll_device_error()
    idx_h = idx.cpu().numpy()
    want = np.stack([oracle.sparse_attn(
        to_f64(data["q"][b]), data["q_pos"][b], q8["kv_cmp"][2][b], idx_h[b], q8["kv_raw"][2][b],
        int(data["raw_pos0"][b]), int(data["n_raw"][b]), data["sink"], wl.scale, wl.window,
        wl.rope_dim, theta_of(wl)) for b in range(wl.B)])
    assert_close(host64(out), want, "bf16", wl.name + " fp8 cache")


def test_csa_decode_fp8_cache():
    # 8 sequences of the 64K-context decode (16,383 entries, top-1,024,
    # 2 tiles of window): several tiles per split, every split
    _check_csa_fp8(W.CSA_DECODE_64K.replace(B=8, seed=91))


def test_csa_decode_fp8_cache_ragged():
    # ragged tiles and fewer visible entries than k
    _check_csa_fp8(W.CSA_DECODE_64K.replace(B=3, T=5003, seed=92))
    _check_csa_fp8(W.CSA_DECODE_64K.replace(B=2, T=2001, seed=93))


def test_hca_decode_fp8_cache():
    wl = W.HCA_DECODE_128K.replace(B=4, seed=94)
    data = W.generate(wl)
    p = params_of(wl)
    q8 = _fp8_caches(data)
    t = {k: dev(data[k]) for k in ("q", "q_pos", "n_cmp", "raw_pos0", "n_raw", "sink")}
    out = torch.empty_like(t["q"])
    nb = csa_workspace_size(p, CSA_OP_HCA_ATTN, wl.B, 1, wl.n_cmp)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    hca_attn_fp8(p, t["q"], t["q_pos"], q8["kv_cmp"][0], q8["kv_cmp"][1], t["n_cmp"],
                 q8["kv_raw"][0], q8["kv_raw"][1], t["raw_pos0"], t["n_raw"], t["sink"], out, ws)
    torch.cuda.synchronize()
    csa_poll_device_error()
    want = np.stack([oracle.hca_attn(
        to_f64(data["q"][b]), data["q_pos"][b], q8["kv_cmp"][2][b], int(data["n_cmp"][b]),
        q8["kv_raw"][2][b], int(data["raw_pos0"][b]), int(data["n_raw"][b]), data["sink"],
        wl.scale, wl.window, wl.width, wl.stride, wl.rope_dim, theta_of(wl))
        for b in range(wl.B)])
    assert_close(host64(out), want, "bf16", "hca fp8 cache")
