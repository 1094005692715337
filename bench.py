#!/usr/bin/env python
"""Benchmark of the CSA layer on B200.

Headline: CSA decode at 64K context, batch 32 (one layer: lightning indexer
+ exact top-1024 + sparse shared-KV attention over 1,024 selected entries
and a 128-token window), in query-heads/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload NAME]

One step = the whole hot path over one batch with the inputs resident in HBM:
decode: indexer scores -> top-k -> sparse attention; HCA decode: dense
attention over every compressed entry; prefill: compression -> indexer ->
top-k -> attention for every token.  Each rank runs an independent replica
of the workload (replicas only: the batch shards with no exchange), so
`scaling` is weak and `value` sums all ranks' query-heads over the slowest
rank's time.  L2 is flushed before every timed step (a 256 MiB write, then a
256 MiB read, so that no dirty line of the flush is left for the step to
write back).  The step runs as one captured CUDA graph timed with CUDA events
on its stream; the per-kernel breakdown comes from a second graph with
events between the launches.  `e2e` runs the same step through the public
layer calls with every step's inputs copied in from pinned host memory and
its result copied out, consecutive steps pipelined on three streams.

`--impl reference` times the fp64 CPU oracle (the only other place this file
runs it) on the host cores, on a bounded sample of the workload per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "csa_decode_bs32_ctx65536"
METRIC = "CSA decode query-heads/s at 64K ctx bs32; % of HBM / bf16 tensor roofline"
UNIT = "query-heads/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TRAFFIC_DIR = os.path.join(ROOT, "profiles")


def _source_digest():
    """Digest of the device code (the kernel headers): recorded DRAM traffic
    is reported only for the kernels it was captured from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_compressed_attention_csa_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith(".cuh"):
            h.update(f.encode())
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def _recorded_traffic(wl):
    """DRAM bytes per launch of each kernel group (dram__bytes_read.sum +
    dram__bytes_write.sum of one ncu capture, profiles/dram_traffic_<workload>
    .json), or {} when absent or captured from other kernel sources."""
    try:
        rec = json.load(open(os.path.join(TRAFFIC_DIR, f"dram_traffic_{wl.name}.json")))
    except (OSError, ValueError):
        return {}
    if rec.get("source_digest") != _source_digest():
        return {}
    return dict(rec.get("bytes_per_launch", {}))


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("cuda", "reference"), default="cuda")
    ap.add_argument("--workload", default=HEADLINE,
                    help="csa_decode_bs32_ctx65536 (default), csa_decode_bs4_ctx1048576, "
                         "hca_decode_bs16_ctx131072, csa_prefill_T8192, "
                         "csa_decode_yarn_bs32_ctx131072, csa2_decode_bs32_ctx65536 "
                         "(one Full + five Reuse layers), hca_prefill_T8192 or "
                         "csa_decode_fp8kv_bs32_ctx65536")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the workload's tokens per sequence (profiling cases)")
    ap.add_argument("--flush-mib", type=int, default=256,
                    help="L2 flush size per side (0: no flush; only for profiling, where the "
                         "profiler flushes caches itself)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def _workload(name, batch=0, seq_len=0):
    from sparse_compressed_attention_csa_b200 import workloads as W
    if name not in W.WORKLOADS or W.WORKLOADS[name].dtype != "bf16":
        raise SystemExit(f"unknown workload {name}; choose from "
                         f"{[n for n, w in W.WORKLOADS.items() if w.dtype == 'bf16']}")
    wl = W.WORKLOADS[name]
    if batch and batch != wl.B:
        wl = wl.replace(B=batch, name=f"{wl.name}_b{batch}")
    if seq_len and seq_len != wl.T:
        wl = wl.replace(T=seq_len, name=f"{wl.name}_T{seq_len}")
    return wl


def _metric(wl):
    return METRIC if wl.name == HEADLINE else f"{wl.name} query-heads/s"


def _config(wl, extra=None, flush_mib=256):
    c = {"workload": wl.name, "kind": wl.kind, "batch": wl.B, "context": wl.T,
         "n_cmp": wl.n_cmp, "query_tokens_per_seq": wl.Tq, "query_heads": wl.n_heads,
         "head_dim": wl.d, "rope_dim": wl.rope_dim, "pool": f"{wl.width}/stride {wl.stride}",
         "window": wl.window,
         "l2": (f"flushed before every timed step: {flush_mib} MiB write, then {flush_mib} MiB read "
                "(L2 left clean)") if flush_mib else "not flushed",
         "parallelism": "replicas"}
    if wl.kind in ("csa_decode", "csa_prefill"):
        c.update({"indexer": f"{wl.idx_heads}x{wl.idx_dim}", "topk": wl.topk})
    if wl.rope_factor > 1.0:
        c["rope"] = (f"theta {wl.theta:g}, YaRN factor {wl.rope_factor:g} over "
                     f"{wl.rope_orig_ctx} tokens")
    if wl.kv_fp8:
        c["kv_cache"] = "E4M3 codes + one fp32 scale per row, quantized after RoPE (outside the step)"
    if wl.reuse_layers:
        c["layers"] = (f"1 Full layer (indexer, top-k, attention) + {wl.reuse_layers} Reuse "
                       "layers (attention over the Full layer's entries and selection)")
    if extra:
        c.update(extra)
    return c


def algorithmic_work(wl):
    """Bytes (and FLOPs) each kernel group of one step must move (do) at
    least, with the inputs resident in HBM, and the whole step's bytes."""
    B, N, H, d, T = wl.B, wl.n_cmp, wl.n_heads, wl.d, wl.T
    Tq = wl.Tq
    n_q = B * Tq
    q = n_q * H * d * 2
    out = n_q * H * d * 2
    if wl.kind == "hca_decode":
        rows = n_q * (N + wl.window) * d * 2
        g = {"hca_attn": {"bytes": rows + q + out + H * 4,
                          "flops": 4 * n_q * H * (N + wl.window) * d}}
        g["step"] = {"bytes": g["hca_attn"]["bytes"]}
        return g
    if wl.kind == "hca_prefill":
        # causal: query t attends to its visible entries and its window
        n_rows = sum(max(0, (t - wl.width) // wl.stride + 1) + min(wl.window, t + 1)
                     for t in range(T))
        g = {"compress": {"bytes": B * T * d * 2 * 2 + B * N * d * 2 + B * T * d * 2,
                          "flops": 0},
             # every entry and raw row read once, q read once, out written once
             "hca_attn": {"bytes": B * (N + T) * d * 2 + q + out + H * 4,
                          "flops": 4 * B * H * n_rows * d}}
        g["step"] = {"bytes": sum(v["bytes"] for v in g.values())}
        return g
    keys = B * N * wl.idx_dim * 2
    idx_q = n_q * wl.idx_heads * (wl.idx_dim * 2 + 4)
    if wl.kind == "csa_decode":
        vis = N                      # every entry is visible to the decode query
        n_rows = min(wl.topk, N) + wl.window
        row_bytes = d + 4 if wl.kv_fp8 else d * 2   # E4M3 codes + scale, or bf16
        rows = n_q * n_rows * row_bytes  # gathered rows (selected + window)
        pre = {}
    else:
        # causal prefill: query t sees floor((t - width) / stride) + 1 entries
        vis = sum(max(0, (t - wl.width) // wl.stride + 1) for t in range(T)) / T
        n_rows = sum(min(wl.topk, max(0, (t - wl.width) // wl.stride + 1)) +
                     min(wl.window, t + 1) for t in range(T)) / T
        rows = B * (N + T) * d * 2   # every pooled entry and raw row read once
        pre = {"compress": {"bytes": B * T * d * 2 * 2 + B * N * d * 2 + B * T * d * 2,
                            "flops": 0}}
    scores = int(n_q * vis) * 4
    sel = n_q * wl.topk * 4
    g = dict(pre)
    g["index_scores"] = {"bytes": keys + idx_q + scores,
                         "flops": int(2 * n_q * vis * wl.idx_heads * wl.idx_dim)}
    g["topk_select"] = {"bytes": scores + sel, "flops": 0}
    g["sparse_attn"] = {"bytes": rows + q + out + sel + H * 4,
                        "flops": int(4 * n_q * H * n_rows * d)}
    if wl.reuse_layers:
        g["reuse_attn"] = {k: wl.reuse_layers * v for k, v in g["sparse_attn"].items()}
    # the step's own bytes: the scores stay between its kernels; the
    # selection is an output of the step (the caller's index buffer), counted
    # once, not again for the attention's read of it (each Reuse layer's read
    # is counted)
    g["step"] = {"bytes": sum(v["bytes"] for v in g.values()) - 2 * scores - sel}
    return g


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock, max clock and clock-event reasons through NVML every
    2 ms on a thread, between start() and stop(), plus one sample as stop()
    is called, so that a short timed region still has several."""
    PERIOD_S = 0.002

    def __init__(self, torch_device):
        self.dev = torch_device
        self.rows = []
        self.stop_evt = threading.Event()
        self.t = None
        self.handle = None
        self.nv = None

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            import torch
            pr = torch.cuda.get_device_properties(self.dev)
            try:
                bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                self.handle = nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.handle = nv.nvmlDeviceGetHandleByIndex(self.dev.index or 0)
        except Exception:
            self.handle = None
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self.handle))

    def _sample(self):
        nv = self.nv
        try:
            self.rows.append((nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM),
                              nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM),
                              self._reasons()))
        except Exception:
            pass

    def _run(self):
        while not self.stop_evt.is_set():
            self._sample()
            time.sleep(self.PERIOD_S)

    def stop(self):
        if self.t is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        self.stop_evt.set()
        self.t.join(timeout=2)
        self._sample()
        bits = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
        reasons = sorted({n for _, _, r in self.rows for n, b in bits.items() if r & b})
        sm = [c for c, _, _ in self.rows]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(m for _, m, _ in self.rows) if self.rows else None,
                "reasons": reasons, "samples": len(sm), "source": "nvml, 2 ms"}


# ------------------------------------------------------------------ oracle arm
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_sample(wl):
    """(step function, query-heads per step, description): the fp64 oracle on
    a bounded sample of the workload."""
    import numpy as np

    import oracle
    from sparse_compressed_attention_csa_b200 import workloads as W
    f = W.to_f64
    v = W.bits_to_f32
    th = wl.theta if wl.rope_factor <= 1.0 else oracle.YaRN(
        theta=wl.theta, factor=wl.rope_factor, orig_ctx=wl.rope_orig_ctx,
        beta_fast=wl.rope_beta_fast, beta_slow=wl.rope_beta_slow)
    if wl.kind == "hca_prefill":
        data = W.generate(wl)
        rows = np.linspace(0, wl.T - 1, 16).astype(np.int64)

        def step():
            kv = oracle.compress(f(data["x"][0]), f(data["g"][0]), wl.width, wl.stride,
                                 wl.rope_dim, th, wl.pos_offset)
            raw = oracle.rotate_raw(f(data["x"][0]), 0, wl.rope_dim, th)
            return oracle.hca_attn(f(data["q"][0][rows]), rows, kv, kv.shape[0], raw, 0, wl.T,
                                   data["sink"], wl.scale, wl.window, wl.width, wl.stride,
                                   wl.rope_dim, th)
        return step, len(rows) * wl.n_heads, (
            "128 -> 1 compression of the whole sequence, then 128-head attention over every "
            "visible entry and the window for 16 of the 8,192 query tokens, fp64 NumPy oracle")
    if wl.kind == "csa_prefill":
        data = W.generate(wl)
        rows = np.linspace(0, wl.T - 1, 16).astype(np.int64)

        def step():
            kv = oracle.compress(f(data["x"][0]), f(data["g"][0]), wl.width, wl.stride,
                                 wl.rope_dim, th, wl.pos_offset)
            raw = oracle.rotate_raw(f(data["x"][0]), 0, wl.rope_dim, th)
            qp = data["q_pos"][0]
            idx = oracle.index_topk(v(data["q_idx"][0]), data["w"][0], f(data["k_idx"][0]), qp,
                                    kv.shape[0], wl.width, wl.stride, wl.topk, rows)
            return oracle.sparse_attn(f(data["q"][0][rows]), qp[rows], kv, idx, raw, 0, wl.T,
                                      data["sink"], wl.scale, wl.window, wl.rope_dim, th)
        return step, len(rows) * wl.n_heads, (
            "compression of the whole sequence, then the indexer, top-k and 128-head attention "
            "for 16 of the 8,192 query tokens, fp64 NumPy oracle")
    one = wl.replace(B=1)  # sequence 0 of the workload: the generator's streams are per tensor
    data = W.generate(one)
    if wl.kind == "hca_decode":
        def step():
            return oracle.hca_attn(f(data["q"][0]), data["q_pos"][0], v(data["kv_cmp"][0]),
                                   int(data["n_cmp"][0]), v(data["kv_raw"][0]),
                                   int(data["raw_pos0"][0]), int(data["n_raw"][0]), data["sink"],
                                   wl.scale, wl.window, wl.width, wl.stride, wl.rope_dim, th)
        return step, wl.n_heads, (f"one of the {wl.B} sequences per step (128-head attention "
                                  f"over its {wl.n_cmp} entries and window), fp64 NumPy oracle")

    kv = {key: v(data[key][0]) for key in ("kv_cmp", "kv_raw")}
    if wl.kv_fp8:  # the caches the quantized ones stand for (quantized outside the step)
        kv = {key: oracle.dequantize_fp8_rows(*oracle.quantize_fp8_rows(val))
              for key, val in kv.items()}

    def attend(q, idx, sink):
        return oracle.sparse_attn(q, data["q_pos"][0], kv["kv_cmp"], idx, kv["kv_raw"],
                                  int(data["raw_pos0"][0]), int(data["n_raw"][0]), sink,
                                  wl.scale, wl.window, wl.rope_dim, th)

    def step():
        qp = data["q_pos"][0]
        idx = oracle.index_topk(f(data["q_idx"][0]), data["w"][0], f(data["k_idx"][0]), qp,
                                int(data["n_cmp"][0]), wl.width, wl.stride, wl.topk)
        outs = [attend(f(data["q"][0]), idx, data["sink"])]
        for r in range(wl.reuse_layers):
            outs.append(attend(f(data["q_reuse"][r][0]), idx, data["sink_reuse"][r]))
        return outs
    reuse = f" + {wl.reuse_layers} Reuse layers" if wl.reuse_layers else ""
    return step, wl.n_heads * (1 + wl.reuse_layers), (
        f"one of the {wl.B} sequences per step (indexer over {wl.n_cmp:,} entries, "
        f"top-{wl.topk}, 128-head attention{reuse}), fp64 NumPy oracle")


def run_reference(args, rank):
    if rank != 0:
        return 0
    wl = _workload(args.workload, args.batch, args.seq_len)
    step, qh, desc = _oracle_sample(wl)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    step()
    t_one = time.perf_counter() - t0
    budget = 150.0
    steps = args.steps if t_one * args.steps <= budget else max(3, int(budget / t_one))
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    el = time.perf_counter() - t0
    value = steps * qh / el
    line = {"impl": "reference", "metric": _metric(wl), "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": steps, "steps_requested": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * el / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def cpu_baseline(wl, budget_s=12.0):
    """The oracle on the sample of `_oracle_sample`, repeated until about
    budget_s of CPU work has elapsed (10-30 s keeps the default run within
    minutes)."""
    step, qh, desc = _oracle_sample(wl)
    t0 = time.perf_counter()
    n = 0
    while True:
        step()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": n * qh / el, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{n} step(s) of: {desc}; {el:.1f} s"}


# ------------------------------------------------------------------ ranks
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's x (all ranks call it, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, slowest_ms: float) -> float:
    """Whole-job throughput of `world` replicas: every rank's units over the
    slowest rank's time (weak scaling)."""
    return world * units_per_rank / (slowest_ms * 1e-3)


# ------------------------------------------------------------------ CUDA arm
def run_cuda(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    from sparse_compressed_attention_csa_b200 import _lib as L
    from sparse_compressed_attention_csa_b200 import build as B
    from sparse_compressed_attention_csa_b200 import layer
    from sparse_compressed_attention_csa_b200 import workloads as W

    B.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl = _workload(args.workload, args.batch, args.seq_len)
    data = W.generate(wl)

    def todev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    t = {k: todev(v) for k, v in data.items()}
    p = L.Params(d=wl.d, rope_dim=wl.rope_dim, theta=wl.theta, scale=wl.scale,
                 n_heads=wl.n_heads, idx_heads=wl.idx_heads, idx_dim=wl.idx_dim, topk=wl.topk,
                 window=wl.window, width=wl.width, stride=wl.stride, pos_offset=wl.pos_offset,
                 rope_factor=wl.rope_factor, rope_orig_ctx=wl.rope_orig_ctx,
                 rope_beta_fast=wl.rope_beta_fast, rope_beta_slow=wl.rope_beta_slow)
    Bsz, Tq, N = wl.B, wl.Tq, wl.n_cmp
    out = torch.empty_like(t["q"])
    hca = wl.kind in ("hca_decode", "hca_prefill")
    prefill = wl.kind in ("csa_prefill", "hca_prefill")
    ops = [L.CSA_OP_HCA_ATTN] if hca else [L.CSA_OP_TOPK_SELECT, L.CSA_OP_SPARSE_ATTN]
    ws_sizes = [L.csa_workspace_size(p, o, Bsz, Tq, N) for o in ops]
    if wl.reuse_layers:  # all Reuse layers in one call: layers x B query rows
        ws_sizes.append(L.csa_workspace_size(p, L.CSA_OP_SPARSE_ATTN, wl.reuse_layers * Bsz, Tq, N))
    ws = torch.empty(max(ws_sizes + [256]), dtype=torch.uint8, device=dev)
    if not hca:
        scores = torch.empty((Bsz, Tq, N), dtype=torch.float32, device=dev)
        idx = torch.empty((Bsz, Tq, wl.topk), dtype=torch.int32, device=dev)
    if wl.kv_fp8:  # the caches as written: quantized after RoPE, once
        for key in ("kv_cmp", "kv_raw"):
            codes, scales = layer.quantize_fp8(t[key])
            t[key + "_fp8"], t[key + "_scale"] = codes, scales
        torch.cuda.synchronize()
    if prefill:
        t["kv_cmp"] = torch.empty((Bsz, N, wl.d), dtype=torch.bfloat16, device=dev)
        t["kv_raw"] = torch.empty((Bsz, wl.T, wl.d), dtype=torch.bfloat16, device=dev)
    if wl.kind == "hca_prefill":
        t["n_cmp"] = torch.full((Bsz,), N, dtype=torch.int32, device=dev)

    # the step's kernel groups, in order
    groups = []
    if prefill:
        groups.append(("compress", lambda: L.csa_compress(p, t["x"], t["g"], t["kv_cmp"],
                                                          t["kv_raw"])))
    if hca:
        groups.append(("hca_attn", lambda: L.hca_attn(
            p, t["q"], t["q_pos"], t["kv_cmp"], t["n_cmp"], t["kv_raw"], t["raw_pos0"],
            t["n_raw"], t["sink"], out, ws)))
    else:
        groups.append(("index_scores", lambda: L.csa_index_scores(
            p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], scores)))
        groups.append(("topk_select", lambda: L.csa_topk_select(
            p, scores, t["q_pos"], t["n_cmp"], idx, ws)))
        if wl.kv_fp8:
            groups.append(("sparse_attn", lambda: L.csa_sparse_attn_fp8(
                p, t["q"], t["q_pos"], t["kv_cmp_fp8"], t["kv_cmp_scale"], idx, t["kv_raw_fp8"],
                t["kv_raw_scale"], t["raw_pos0"], t["n_raw"], t["sink"], out, ws)))
        else:
            groups.append(("sparse_attn", lambda: L.csa_sparse_attn(
                p, t["q"], t["q_pos"], t["kv_cmp"], idx, t["kv_raw"], t["raw_pos0"], t["n_raw"],
                t["sink"], out, ws)))
    R = wl.reuse_layers
    if R:
        out_r = torch.empty_like(t["q_reuse"])

        groups.append(("reuse_attn", lambda: L.csa_reuse_attn(
            p, t["q_reuse"], t["q_pos"], t["kv_cmp"], idx, t["kv_raw"], t["raw_pos0"],
            t["n_raw"], t["sink_reuse"], out_r, ws)))

    mib = max(args.flush_mib, 0)
    flush = torch.empty(mib << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(mib << 18, dtype=torch.float32, device=dev)

    def flush_l2():
        if mib:
            flush.zero_()
            flush_rd.sum()  # evicts the dirty lines of the write: L2 left clean
    stream = torch.cuda.Stream(device=dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(groups) + 1)]

    def launch(marks=False):
        # marks: events between the kernels, for the per-kernel breakdown
        # (they cut the programmatic-launch overlap, so the timed step has none)
        for i, (_, fn) in enumerate(groups):
            if marks:
                ev[i].record()
            fn()
        if marks:
            ev[len(groups)].record()

    with torch.cuda.stream(stream):
        n0 = L.csa_launch_count()
        launch()  # eager warm-up (module load, attribute setup)
        kernels_per_step = L.csa_launch_count() - n0
    torch.cuda.synchronize()
    L.csa_poll_device_error(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        launch()
    graph_marked = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_marked, stream=stream):
        launch(marks=True)
    torch.cuda.synchronize()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)

    def timed_steps(n):
        tot = 0.0
        for _ in range(n):
            with torch.cuda.stream(stream):
                flush_l2()
                s0.record()
                graph.replay()
                s1.record()
            stream.synchronize()
            tot += s0.elapsed_time(s1)
        return tot

    def breakdown(n):
        tot = [0.0] * len(groups)
        for _ in range(n):
            with torch.cuda.stream(stream):
                flush_l2()
                graph_marked.replay()
            stream.synchronize()
            for i in range(len(groups)):
                tot[i] += ev[i].elapsed_time(ev[i + 1])
        return [x / n for x in tot]

    timed_steps(args.warmup)
    sampler = ClockSampler(dev) if not args.no_clocks else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    tot = timed_steps(args.steps)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    L.csa_poll_device_error(stream)

    step_ms = tot / args.steps
    n_bd = min(args.steps, 200)
    bd = breakdown(n_bd)
    step_ms_max = max_over_ranks(step_ms, world, dev)
    qh_per_step = wl.B * wl.Tq * wl.n_heads * (1 + R)
    value = job_throughput(qh_per_step, world, step_ms_max)

    # end to end through the public API: pinned host inputs -> device -> layer -> host.
    # Throughput is measured the way a serving loop runs consecutive steps:
    # step i's inputs go host -> device on one stream while step i - 1
    # computes on a second and step i - 2's result goes device -> host on a
    # third (PCIe carries both directions at once), two sets of device inputs
    # and outputs alternating.  Every step copies its own inputs in and its
    # own result out inside the timed region.  The latency of one step on its
    # own (copy in, compute, copy out in sequence) is reported beside it.
    h2d_keys = {"csa_decode": ("q", "q_idx", "w", "q_pos"), "hca_decode": ("q", "q_pos"),
                "csa_prefill": ("x", "g", "q_idx", "w", "q"),
                "hca_prefill": ("x", "g", "q")}[wl.kind] + (("q_reuse",) if R else ())
    h_in = {k: torch.from_numpy(np.ascontiguousarray(data[k].view(np.int16) if data[k].dtype ==
                                                      np.uint16 else data[k])).pin_memory()
            for k in h2d_keys}
    NBUF = 2
    d_ins = [{k: torch.empty(h_in[k].shape, dtype=h_in[k].dtype, device=dev) for k in h_in}
             for _ in range(NBUF)]
    outs = [out] + [torch.empty_like(out) for _ in range(NBUF - 1)]
    outs_r = ([out_r] + [torch.empty_like(out_r) for _ in range(NBUF - 1)]) if R else None
    h_outs = [[torch.empty(out.shape, dtype=torch.int16).pin_memory()]
              + ([torch.empty(out_r.shape, dtype=torch.int16).pin_memory()] if R else [])
              for _ in range(NBUF)]
    lw = layer.Workspace(dev)
    h2d = sum(h_in[k].numel() * h_in[k].element_size() for k in h_in)
    d2h = sum(h.numel() * h.element_size() for h in h_outs[0])

    # a step whose resident reads fit in the L2 cycles through copies of its
    # caches (together more than twice the L2), so that no step finds its
    # caches there; a larger one reads the same caches every step
    L2_BYTES = 126 * 2 ** 20
    step_bytes = algorithmic_work(wl)["step"]["bytes"]
    n_sets = 1 if step_bytes > L2_BYTES else -(-2 * L2_BYTES // step_bytes)
    resident = [k for k in ("k_idx", "kv_cmp", "kv_raw", "kv_cmp_fp8", "kv_cmp_scale",
                            "kv_raw_fp8", "kv_raw_scale") if k in t]
    t_sets = [t] + [dict(t, **{k: t[k].clone() for k in resident}) for _ in range(n_sets - 1)]

    def run_layer(d, j, c=0):
        """One step through the public layer calls on the current stream,
        on input buffers d, output set j and cache copy c; returns the
        result tensors to read back."""
        t = t_sets[c]

        def bf(k):
            return d[k].view(torch.bfloat16)
        if wl.kind == "csa_decode" and wl.kv_fp8:
            _, o = layer.csa_decode_fp8(
                p, bf("q"), d["q_pos"], bf("q_idx"), d["w"], t["k_idx"], t["n_cmp"],
                t["kv_cmp_fp8"], t["kv_cmp_scale"], t["kv_raw_fp8"], t["kv_raw_scale"],
                t["raw_pos0"], t["n_raw"], t["sink"], lw, idx=idx, out=outs[j])
            return [o]
        if wl.kind == "csa_decode":
            _, o = layer.csa_decode(p, bf("q"), d["q_pos"], bf("q_idx"), d["w"], t["k_idx"],
                                    t["n_cmp"], t["kv_cmp"], t["kv_raw"], t["raw_pos0"],
                                    t["n_raw"], t["sink"], lw, idx=idx, out=outs[j])
            if not R:
                return [o]
            layer.reuse_attn(p, bf("q_reuse"), d["q_pos"], t["kv_cmp"], idx, t["kv_raw"],
                             t["raw_pos0"], t["n_raw"], t["sink_reuse"], lw, out=outs_r[j])
            return [o, outs_r[j]]
        if wl.kind == "hca_decode":
            return [layer.hca_decode(p, bf("q"), d["q_pos"], t["kv_cmp"], t["n_cmp"], t["kv_raw"],
                                     t["raw_pos0"], t["n_raw"], t["sink"], lw, out=outs[j])]
        if wl.kind == "hca_prefill":
            return [layer.hca_prefill(p, bf("x"), bf("g"), bf("q"), t["sink"], lw, out=outs[j])[2]]
        return [layer.csa_prefill(p, bf("x"), bf("g"), bf("q_idx"), d["w"], t["k_idx"], bf("q"),
                                  t["sink"], lw)[3]]

    def read_back(res, j, s_copy):
        for r, h in zip(res, h_outs[j]):
            h.copy_(r.view(torch.int16), non_blocking=True)
            r.record_stream(s_copy)  # a result the layer allocated outlives its step

    def e2e_latency_step():
        with torch.cuda.stream(stream):
            flush_l2()
            e_start.record()
            for k in h_in:
                d_ins[0][k].copy_(h_in[k], non_blocking=True)
            read_back(run_layer(d_ins[0], 0), 0, stream)
            e_end.record()
        stream.synchronize()
        return e_start.elapsed_time(e_end)

    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    in_done = [torch.cuda.Event() for _ in range(NBUF)]
    cmp_done = [torch.cuda.Event() for _ in range(NBUF)]
    out_done = [torch.cuda.Event() for _ in range(NBUF)]

    host_s = [0.0]

    def e2e_pipelined(n):
        main = torch.cuda.current_stream()
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        e_start.record(main)
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_event(e_start)
        # (set_stream rather than the stream context manager: the same effect
        # at a fraction of the host cost per switch)
        for i in range(n):
            j = i % NBUF
            torch.cuda.set_stream(s_in)
            if i >= NBUF:
                s_in.wait_event(cmp_done[j])  # step i - 2 is done with these inputs
            for k in h_in:
                d_ins[j][k].copy_(h_in[k], non_blocking=True)
            in_done[j].record(s_in)
            torch.cuda.set_stream(s_cmp)
            s_cmp.wait_event(in_done[j])
            if i >= NBUF:
                s_cmp.wait_event(out_done[j])  # step i - 2's result has been read
            res = run_layer(d_ins[j], j, i % n_sets)
            cmp_done[j].record(s_cmp)
            torch.cuda.set_stream(s_out)
            s_out.wait_event(cmp_done[j])
            read_back(res, j, s_out)
            out_done[j].record(s_out)
        torch.cuda.set_stream(main)
        main.wait_stream(s_out)
        e_end.record(main)
        host_s[0] = time.perf_counter() - h0  # the host's enqueue time for the n steps
        e_end.synchronize()
        return e_start.elapsed_time(e_end) / n

    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    n_e2e = max(20, min(args.steps, 200))
    n_lat = max(10, min(args.steps, 50))
    for _ in range(max(args.warmup, 5)):
        e2e_latency_step()
    lat_ms = sum(e2e_latency_step() for _ in range(n_lat)) / n_lat
    e2e_pipelined(max(args.warmup, 10))
    if world > 1:
        dist.barrier()
    e2e_ms = e2e_pipelined(n_e2e)
    e2e_value = job_throughput(qh_per_step, world, max_over_ranks(e2e_ms, world, dev))
    lat_ms = max_over_ranks(lat_ms, world, dev)
    if world > 1:
        dist.barrier()
    L.csa_poll_device_error(stream)

    if rank == 0:
        peaks = {}
        if os.path.exists(PEAKS_FILE):
            peaks = json.load(open(PEAKS_FILE))
        src = "measured" if peaks else "fallback"
        hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        tc = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        work = algorithmic_work(wl)
        kernel_ms = {name: bd[i] for i, (name, _) in enumerate(groups)}
        traffic = _recorded_traffic(wl)
        rl = {}
        for k, ms in kernel_ms.items():
            b, f = work[k]["bytes"], work[k]["flops"]
            gbs = b / (ms * 1e-3) / 1e9
            tfl = f / (ms * 1e-3) / 1e12
            # the bound is the roof that the kernel's arithmetic intensity meets first
            tensor = f > 0 and f / b > tc * 1e12 / (hbm * 1e9)
            rl[k] = {"bound": "tensor" if tensor else "hbm",
                     "achieved": tfl if tensor else gbs, "peak": tc if tensor else hbm,
                     "unit": "TFLOP/s" if tensor else "GB/s",
                     "frac": (tfl / tc) if tensor else (gbs / hbm),
                     "algorithmic_bytes": b, "flops": f, "ms": ms,
                     "hbm_frac": gbs / hbm, "tensor_frac": tfl / tc if f else 0.0,
                     "traffic": traffic.get(k), "peak_source": src + " burst"}
        dom = max(kernel_ms, key=kernel_ms.get)
        line = {
            "metric": _metric(wl), "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": _config(wl, flush_mib=mib),
            "gpu_launches": kernels_per_step * args.steps,
            "kernels_per_step": kernels_per_step,
            "kernel_ms": kernel_ms,
            "kernel_ms_note": f"{n_bd} steps of the same graph with events between the launches "
                              "(no programmatic-launch overlap there); the timed step has none",
            "step_hbm": {"algorithmic_bytes": work["step"]["bytes"],
                         "achieved_gbs": work["step"]["bytes"] / (step_ms_max * 1e-3) / 1e9,
                         "frac": work["step"]["bytes"] / (step_ms_max * 1e-3) / 1e9 / hbm,
                         "peak_source": src},
            "roofline": dict(kernel=dom, **{k: v for k, v in rl[dom].items()
                                            if k in ("bound", "achieved", "peak", "unit", "frac",
                                                     "traffic", "peak_source")}),
            "roofline_by_kernel": rl,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": n_e2e, "ms_per_step": e2e_ms,
                    "mode": "consecutive steps pipelined on three streams (copy in, layer calls, "
                            "copy out), two buffer sets",
                    "l2": (f"not flushed: a step reads {step_bytes / 1e6:.0f} MB resident in "
                           "HBM, more than the 126 MB L2" if n_sets == 1 else
                           f"not flushed: consecutive steps cycle through {n_sets} copies of the "
                           f"resident caches ({n_sets * step_bytes / 1e6:.0f} MB, more than "
                           "twice the 126 MB L2)"),
                    "host_enqueue_ms_per_step": host_s[0] * 1e3 / n_e2e,
                    "latency_ms": lat_ms,
                    "latency_note": "one step alone: copy in, layer calls, copy out in sequence "
                                    "on one stream, L2 flushed before it (untimed)"},
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line))
    del graph, graph_marked
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = _args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    return run_cuda(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
