#!/usr/bin/env python
"""Benchmark of the CSA decode layer on B200: query-heads/s at 64K context,
batch 32 (one layer: lightning indexer + exact top-1024 + sparse shared-KV
attention over 1,024 selected entries and a 128-token window).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

One step = the whole decode hot path over one batch (32 sequences x 1 query
token x 128 heads) with the caches resident in HBM.  Each rank runs an
independent replica of the workload (replicas only: the decode batch
shards with no exchange), so `scaling` is weak and `value` sums all ranks'
query-heads over the slowest rank's time.  L2 is flushed (a 256 MiB write)
before every timed step; each step is a captured CUDA graph whose per-kernel
durations come from CUDA events recorded inside it.

`--impl reference` times the fp64 CPU oracle (the only other place this file
runs it) on the host cores, one sequence per step.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA decode query-heads/s at 64K ctx bs32; % of HBM / bf16 tensor roofline"
UNIT = "query-heads/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("cuda", "reference"), default="cuda")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def _workload():
    from sparse_compressed_attention_csa_b200 import workloads as W
    return W.CSA_DECODE_64K


def _config(wl, extra=None):
    c = {"workload": wl.name, "batch": wl.B, "context": wl.T, "n_cmp": wl.n_cmp,
         "query_heads": wl.n_heads, "head_dim": wl.d, "rope_dim": wl.rope_dim,
         "indexer": f"{wl.idx_heads}x{wl.idx_dim}", "topk": wl.topk, "window": wl.window,
         "l2": "flushed (256 MiB write) before every timed step", "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


def algorithmic_bytes(wl):
    """Bytes one decode step must move at least (caches resident)."""
    B, N, H, d = wl.B, wl.n_cmp, wl.n_heads, wl.d
    keys = B * N * wl.idx_dim * 2
    idx_q = B * wl.idx_heads * wl.idx_dim * 2 + B * wl.idx_heads * 4
    rows = B * (min(wl.topk, N) + wl.window) * d * 2
    q = B * H * d * 2
    out = B * H * d * 2
    small = B * wl.topk * 4 + H * 4
    return {"index_scores": keys + idx_q + B * N * 4, "step": keys + idx_q + rows + q + out + small}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.lines: list[str] = []
        self.proc = None
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        deadline = time.time() + 5
        while not self.lines and time.time() < deadline:
            time.sleep(0.02)
        self.mark = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        end = len(self.lines)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [l.split(", ") for l in self.lines[self.mark:end] if l]
        sm = [float(r[1]) for r in rows if len(r) > 8 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) > 8 and r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            if len(r) > 8:
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank):
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from sparse_compressed_attention_csa_b200 import workloads as W
    wl = _workload()
    one = wl.replace(B=1)  # sequence 0 of the workload: the generator's streams are per tensor
    data = W.generate(one)
    f = W.to_f64

    def step():
        qp = data["q_pos"][0]
        idx = oracle.index_topk(f(data["q_idx"][0]), data["w"][0], f(data["k_idx"][0]), qp,
                                int(data["n_cmp"][0]), wl.width, wl.stride, wl.topk)
        return oracle.sparse_attn(f(data["q"][0]), qp, W.bits_to_f32(data["kv_cmp"][0]), idx,
                                  W.bits_to_f32(data["kv_raw"][0]), int(data["raw_pos0"][0]),
                                  int(data["n_raw"][0]), data["sink"], wl.scale, wl.window,
                                  wl.rope_dim, wl.theta)

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
    value = steps * wl.n_heads / el
    cores = _blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "one of the 32 sequences per step (its indexer, top-k and "
                                       "128-head attention), fp64 NumPy oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=12.0):
    """The oracle on whole sequences of the workload, until ~budget_s elapsed."""
    import oracle
    from sparse_compressed_attention_csa_b200 import workloads as W
    one = wl.replace(B=1)
    data = W.generate(one)
    f = W.to_f64
    t0 = time.perf_counter()
    n = 0
    while True:
        qp = data["q_pos"][0]
        idx = oracle.index_topk(f(data["q_idx"][0]), data["w"][0], f(data["k_idx"][0]), qp,
                                int(data["n_cmp"][0]), wl.width, wl.stride, wl.topk)
        oracle.sparse_attn(f(data["q"][0]), qp, W.bits_to_f32(data["kv_cmp"][0]), idx,
                           W.bits_to_f32(data["kv_raw"][0]), int(data["raw_pos0"][0]),
                           int(data["n_raw"][0]), data["sink"], wl.scale, wl.window, wl.rope_dim,
                           wl.theta)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 64:
            break
    return {"value": n * wl.n_heads / el, "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{n} whole sequence(s) of the workload (indexer over 16,383 entries, "
                      f"top-1024, 128-head attention), fp64 NumPy, {el:.1f} s"}


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
    wl = _workload()
    data = W.generate(wl)

    def todev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    t = {k: todev(v) for k, v in data.items()}
    p = L.Params(topk=wl.topk, window=wl.window)
    Bsz, Tq, N = wl.B, 1, wl.n_cmp
    scores = torch.empty((Bsz, Tq, N), dtype=torch.float32, device=dev)
    idx = torch.empty((Bsz, Tq, wl.topk), dtype=torch.int32, device=dev)
    out = torch.empty_like(t["q"])
    ws_topk = L.csa_workspace_size(p, L.CSA_OP_TOPK_SELECT, Bsz, Tq, N)
    ws_attn = L.csa_workspace_size(p, L.CSA_OP_SPARSE_ATTN, Bsz, Tq, N)
    ws = torch.empty(max(ws_topk, ws_attn, 256), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]

    def launch():
        ev[0].record()
        L.csa_index_scores(p, t["q_idx"], t["w"], t["k_idx"], t["q_pos"], t["n_cmp"], scores)
        ev[1].record()
        L.csa_topk_select(p, scores, t["q_pos"], t["n_cmp"], idx, ws)
        ev[2].record()
        L.csa_sparse_attn(p, t["q"], t["q_pos"], t["kv_cmp"], idx, t["kv_raw"], t["raw_pos0"],
                          t["n_raw"], t["sink"], out, ws)
        ev[3].record()

    kernels_per_step = 3
    with torch.cuda.stream(stream):
        launch()  # eager warm-up (module load, attribute setup)
    torch.cuda.synchronize()
    L.csa_poll_device_error(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        launch()
    torch.cuda.synchronize()

    def timed_steps(n):
        tot = [0.0, 0.0, 0.0, 0.0]
        for _ in range(n):
            with torch.cuda.stream(stream):
                flush.zero_()
                graph.replay()
            stream.synchronize()
            a, b, c = (ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]),
                       ev[2].elapsed_time(ev[3]))
            tot[0] += a + b + c
            tot[1] += a
            tot[2] += b
            tot[3] += c
        return tot

    timed_steps(args.warmup)
    sampler = ClockSampler(local) if not args.no_clocks else None
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

    step_ms = tot[0] / args.steps
    t_max = torch.tensor([step_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_max, op=dist.ReduceOp.MAX)
    step_ms_max = float(t_max.item())
    qh_per_step = wl.B * wl.n_heads
    value = world * qh_per_step / (step_ms_max * 1e-3)

    # end to end through the public API: pinned host inputs -> device -> layer -> host
    h_in = {k: torch.from_numpy(np.ascontiguousarray(data[k].view(np.int16) if data[k].dtype ==
                                                      np.uint16 else data[k])).pin_memory()
            for k in ("q", "q_idx", "w", "q_pos")}
    d_in = {k: torch.empty(h_in[k].shape, dtype=h_in[k].dtype, device=dev) for k in h_in}
    h_out = torch.empty(out.shape, dtype=torch.int16).pin_memory()
    lw = layer.Workspace(dev)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    h2d = sum(h_in[k].numel() * h_in[k].element_size() for k in h_in)
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        with torch.cuda.stream(stream):
            flush.zero_()
            e_start.record()
            for k in h_in:
                d_in[k].copy_(h_in[k], non_blocking=True)
            q = d_in["q"].view(torch.bfloat16)
            qi = d_in["q_idx"].view(torch.bfloat16)
            _, o = layer.csa_decode(p, q, d_in["q_pos"], qi, d_in["w"], t["k_idx"], t["n_cmp"],
                                    t["kv_cmp"], t["kv_raw"], t["raw_pos0"], t["n_raw"],
                                    t["sink"], lw, idx=idx, out=out)
            h_out.copy_(o.view(torch.int16), non_blocking=True)
            e_end.record()
        stream.synchronize()
        return e_start.elapsed_time(e_end)

    for _ in range(args.warmup):
        e2e_step()
    if world > 1:
        dist.barrier()
    e2e_ms = sum(e2e_step() for _ in range(args.steps)) / args.steps
    e_max = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e_max, op=dist.ReduceOp.MAX)
        dist.barrier()
    e2e_value = world * qh_per_step / (float(e_max.item()) * 1e-3)

    if rank == 0:
        peaks = {}
        if os.path.exists(PEAKS_FILE):
            peaks = json.load(open(PEAKS_FILE))
        hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        ab = algorithmic_bytes(wl)
        t_scores = tot[1] / args.steps * 1e-3
        achieved = ab["index_scores"] / t_scores / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": _config(wl),
            "gpu_launches": kernels_per_step * args.steps,
            "kernel_ms": {"index_scores": tot[1] / args.steps, "topk_select": tot[2] / args.steps,
                          "sparse_attn": tot[3] / args.steps},
            "step_hbm": {"algorithmic_bytes": ab["step"],
                         "achieved_gbs": ab["step"] / (step_ms_max * 1e-3) / 1e9,
                         "frac_of_measured": ab["step"] / (step_ms_max * 1e-3) / 1e9 / hbm},
            "roofline": {"kernel": "index_scores", "bound": "hbm", "achieved": achieved,
                         "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "peak_source": "measured" if peaks else "fallback",
                         "traffic": None},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line))
    del graph
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
