#!/usr/bin/env python
"""Benchmark of the CSA decode layer on B200: query-heads/s at 64K context,
batch 32 (one layer: lightning indexer + exact top-1024 + sparse shared-KV
attention over 1,024 selected entries and a 128-token window).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

One step = the whole decode hot path over one batch (32 sequences x 1 query
token x 128 heads) with the caches resident in HBM.  Each rank runs an
independent replica of the workload (replicas only: the decode batch
shards with no exchange), so `scaling` is weak and `value` sums all ranks'
query-heads over the slowest rank's time.  L2 is flushed before every timed
step (a 256 MiB write, then a 256 MiB read, so that no dirty line of the
flush is left for the step to write back); each step is a captured CUDA graph
whose per-kernel durations come from CUDA events recorded inside it.

`--impl reference` times the fp64 CPU oracle (the only other place this file
runs it) on the host cores, one sequence per step.
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

METRIC = "CSA decode query-heads/s at 64K ctx bs32; % of HBM / bf16 tensor roofline"
UNIT = "query-heads/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_csa_decode_bs32_ctx65536.json")


def _source_digest():
    """Digest of the kernel sources: recorded DRAM traffic is only reported
    for the kernels it was captured from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_compressed_attention_csa_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def _recorded_traffic(wl):
    """DRAM bytes per launch group (dram__bytes_read.sum + dram__bytes_write.sum
    from one ncu capture of this workload), or {} if the kernels changed."""
    try:
        rec = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return {}
    if rec.get("source_digest") != _source_digest() or rec.get("workload") != wl.name:
        return {}
    return {k: v for k, v in rec.get("bytes_per_launch", {}).items()}


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
         "l2": "flushed before every timed step: 256 MiB write, then 256 MiB read (L2 left clean)",
         "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


def algorithmic_work(wl):
    """Bytes (and FLOPs) one decode step must move (do) at least, per kernel
    group and for the whole step, with the caches resident in HBM."""
    B, N, H, d = wl.B, wl.n_cmp, wl.n_heads, wl.d
    keys = B * N * wl.idx_dim * 2
    idx_q = B * wl.idx_heads * wl.idx_dim * 2 + B * wl.idx_heads * 4
    scores = B * N * 4
    sel = B * wl.topk * 4
    n_rows = min(wl.topk, N) + wl.window
    rows = B * n_rows * d * 2
    q = B * H * d * 2
    out = B * H * d * 2
    return {
        "index_scores": {"bytes": keys + idx_q + scores, "flops": 2 * B * N * wl.idx_heads * wl.idx_dim},
        "topk_select": {"bytes": scores + sel, "flops": 0},
        "sparse_attn": {"bytes": rows + q + out + sel + H * 4, "flops": 4 * B * H * n_rows * d},
        "step": {"bytes": keys + idx_q + rows + q + out + sel + H * 4},
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock, max clock and clock-event reasons through NVML every
    20 ms on a thread, between start() and stop()."""
    PERIOD_S = 0.02

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

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                self.rows.append((nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM),
                                  nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM),
                                  self._reasons()))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def stop(self):
        if self.t is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        self.stop_evt.set()
        self.t.join(timeout=2)
        bits = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
        reasons = sorted({n for _, _, r in self.rows for n, b in bits.items() if r & b})
        sm = [c for c, _, _ in self.rows]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(m for _, m, _ in self.rows) if self.rows else None,
                "reasons": reasons, "samples": len(sm), "source": "nvml, 20 ms"}


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
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)  # 256 MiB

    def flush_l2():
        flush.zero_()
        flush_rd.sum()  # evicts the dirty lines of the write: L2 left clean
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

    with torch.cuda.stream(stream):
        n0 = L.csa_launch_count()
        launch()  # eager warm-up (module load, attribute setup)
        kernels_per_step = L.csa_launch_count() - n0
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
                flush_l2()
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
            flush_l2()
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
        src = "measured" if peaks else "fallback"
        hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        tc = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        work = algorithmic_work(wl)
        kernel_ms = {"index_scores": tot[1] / args.steps, "topk_select": tot[2] / args.steps,
                     "sparse_attn": tot[3] / args.steps}
        traffic = _recorded_traffic(wl)
        rl = {}
        for k, ms in kernel_ms.items():
            b, f = work[k]["bytes"], work[k]["flops"]
            gbs = b / (ms * 1e-3) / 1e9
            tfl = f / (ms * 1e-3) / 1e12
            # the bound is the roof the kernel's arithmetic intensity meets first
            tensor = f > 0 and f / b > tc * 1e12 / (hbm * 1e9)
            rl[k] = {"bound": "tensor" if tensor else "hbm",
                     "achieved": tfl if tensor else gbs, "peak": tc if tensor else hbm,
                     "unit": "TFLOP/s" if tensor else "GB/s",
                     "frac": (tfl / tc) if tensor else (gbs / hbm),
                     "algorithmic_bytes": b, "flops": f, "ms": ms,
                     "tensor_frac": tfl / tc if f else 0.0,
                     "traffic": traffic.get(k), "peak_source": src + " burst"}
        dom = max(kernel_ms, key=kernel_ms.get)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": _config(wl),
            "gpu_launches": kernels_per_step * args.steps,
            "kernels_per_step": kernels_per_step,
            "kernel_ms": kernel_ms,
            "step_hbm": {"algorithmic_bytes": work["step"]["bytes"],
                         "achieved_gbs": work["step"]["bytes"] / (step_ms_max * 1e-3) / 1e9,
                         "frac": work["step"]["bytes"] / (step_ms_max * 1e-3) / 1e9 / hbm,
                         "peak_source": src},
            "roofline": dict(kernel=dom, **{k: v for k, v in rl[dom].items()
                                            if k in ("bound", "achieved", "peak", "unit", "frac",
                                                     "traffic", "peak_source")}),
            "roofline_by_kernel": rl,
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
