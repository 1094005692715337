"""Helpers shared by the GPU tests: move generated inputs to the device,
run the layer through the C-ABI binding, compare with the oracle."""
import json
import os

import numpy as np
import torch

from sparse_compressed_attention_csa_b200 import Params, layer
from sparse_compressed_attention_csa_b200.workloads import Workload, to_f64

# Acceptance bounds: bit-exact indices; bf16 max-abs 2e-2 and relative L2
# 5e-3; fp32 1e-5 for both.
TOL = {"bf16": (2e-2, 5e-3), "f32": (1e-5, 1e-5)}


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def params_of(wl: Workload) -> Params:
    return Params(d=wl.d, rope_dim=wl.rope_dim, theta=wl.theta, scale=wl.scale,
                  n_heads=wl.n_heads, idx_heads=wl.idx_heads, idx_dim=wl.idx_dim, topk=wl.topk,
                  window=wl.window, width=wl.width, stride=wl.stride, pos_offset=wl.pos_offset,
                  rope_factor=wl.rope_factor, rope_orig_ctx=wl.rope_orig_ctx,
                  rope_beta_fast=wl.rope_beta_fast, rope_beta_slow=wl.rope_beta_slow)


def theta_of(wl: Workload):
    """The oracle's RoPE argument for a workload: the base, or a YaRN spec."""
    import oracle
    if wl.rope_factor > 1.0:
        return oracle.YaRN(theta=wl.theta, factor=wl.rope_factor, orig_ctx=wl.rope_orig_ctx,
                           beta_fast=wl.rope_beta_fast, beta_slow=wl.rope_beta_slow)
    return wl.theta


def assert_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = ""):
    tol_abs, tol_rel = TOL[dtype]
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.max(np.abs(got - want))) if got.size else 0.0
    nrm = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(got - want)) / nrm if nrm > 0 else err
    log = os.environ.get("CSA_ERRLOG")  # optional record of every comparison's error
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"what": what, "dtype": dtype, "max_abs": err, "rel_l2": rel}) + "\n")
    assert err <= tol_abs and rel <= tol_rel, f"{what}: max-abs {err:.3e} rel-L2 {rel:.3e}"
    return err, rel


def run_decode(wl: Workload, data: dict):
    p = params_of(wl)
    t = {k: dev(v) for k, v in data.items()}
    idx, out = layer.csa_decode(p, t["q"], t["q_pos"], t["q_idx"], t["w"], t["k_idx"],
                                t["n_cmp"], t["kv_cmp"], t["kv_raw"], t["raw_pos0"], t["n_raw"],
                                t["sink"])
    torch.cuda.synchronize()
    return idx, out


def run_hca(wl: Workload, data: dict):
    p = params_of(wl)
    t = {k: dev(v) for k, v in data.items()}
    out = layer.hca_decode(p, t["q"], t["q_pos"], t["kv_cmp"], t["n_cmp"], t["kv_raw"],
                           t["raw_pos0"], t["n_raw"], t["sink"])
    torch.cuda.synchronize()
    return out


def run_prefill(wl: Workload, data: dict):
    p = params_of(wl)
    t = {k: dev(v) for k, v in data.items()}
    kv_cmp, kv_raw, idx, out = layer.csa_prefill(p, t["x"], t["g"], t["q_idx"], t["w"],
                                                 t["k_idx"], t["q"], t["sink"])
    torch.cuda.synchronize()
    return kv_cmp, kv_raw, idx, out


def f64(data: dict, key: str, *index):
    a = data[key]
    if index:
        a = a[index]
    return to_f64(a)
