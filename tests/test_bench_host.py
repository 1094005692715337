"""The bench's roofline numerators: algorithmic bytes and FLOPs of one step,
checked against totals derived by hand from the workloads' shapes (no GPU).

Bytes count what a step must move with its inputs resident in HBM; FLOPs
are the multiply-adds x 2 of the two contractions (indexer q.k over the
visible entries; attention q.k and p.v over the gathered rows).
"""
import bench
from sparse_compressed_attention_csa_b200 import workloads as W

KB = 1024


def test_headline_decode_bytes_and_flops():
    # 32 sequences, 16,383 entries, top-1,024 + a 128-row window, 128 heads x 512
    keys = 32 * 16383 * 256              # indexer keys, 128 bf16 each
    rows = 32 * 1152 * KB                # gathered rows: 1,024 selected + 128 window, 1 KB each
    q = out = 32 * 128 * KB              # 128 heads x 512 bf16 per token, in and out
    q_idx, w = 32 * 64 * 256, 32 * 64 * 4
    sel = 32 * 1024 * 4                  # the selection, an output of the step
    sink = 128 * 4
    g = bench.algorithmic_work(W.CSA_DECODE_64K)
    assert keys + rows + q + out + q_idx + w + sel + sink == 181_010_944
    assert g["step"]["bytes"] == 181_010_944
    assert g["sparse_attn"]["bytes"] == rows + q + out + sel + sink == 46_268_928
    assert g["index_scores"]["flops"] == 2 * 32 * 16383 * 64 * 128
    assert g["sparse_attn"]["flops"] == 4 * 32 * 128 * 1152 * 512
    assert g["index_scores"]["flops"] + g["sparse_attn"]["flops"] == 18_253_086_720


def test_long_context_decode_bytes():
    # 4 sequences of 262,143 entries: the indexer keys dominate
    total = (4 * 262143 * 256 + 4 * 1152 * KB + 2 * 4 * 128 * KB + 4 * 64 * 256 + 4 * 64 * 4
             + 4 * 1024 * 4 + 128 * 4)
    assert total == 274_285_056
    assert bench.algorithmic_work(W.CSA_DECODE_1M)["step"]["bytes"] == total


def test_hca_decode_bytes_and_flops():
    # 16 tokens over all 1,024 entries + the window: no indexer, no selection
    g = bench.algorithmic_work(W.HCA_DECODE_128K)
    assert g["step"]["bytes"] == 16 * 1152 * KB + 2 * 16 * 128 * KB + 128 * 4 == 23_069_184
    assert g["hca_attn"]["flops"] == 4 * 16 * 128 * 1152 * 512 == 4_831_838_208


def test_prefill_flops():
    # causal: token t sees floor((t - 8) / 4) + 1 entries (at most 1,024
    # selected) and min(128, t + 1) window rows
    T = 8192
    vis = [max(0, (t - 8) // 4 + 1) for t in range(T)]
    rows = sum(min(1024, v) + min(128, t + 1) for t, v in enumerate(vis))
    g = bench.algorithmic_work(W.CSA_PREFILL_8K)
    assert g["sparse_attn"]["flops"] == 4 * 128 * rows * 512
    assert g["index_scores"]["flops"] == 2 * sum(vis) * 64 * 128
    assert round((g["sparse_attn"]["flops"] + g["index_scores"]["flops"]) / 1e12, 3) == 2.058


def _run_bench(args, env_extra=None, timeout=300):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root, env=env,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    return lines


def test_reference_arm_prints_one_complete_line():
    # the oracle timed on the host cores on the headline's config: one JSON
    # line with the same metric, unit and direction as the CUDA arm, its own
    # cpu_baseline, and an e2e entry that moves no bytes
    (line,) = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3"])
    assert line["impl"] == "reference"
    assert line["unit"] == "query-heads/s" and line["higher_is_better"] is True
    assert line["metric"].startswith("CSA decode query-heads/s")
    assert line["config"]["workload"] == "csa_decode_bs32_ctx65536"
    assert line["value"] > 0 and line["dtype"] == "f64" and line["warmup"] >= 3
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "query-heads/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    assert _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3"],
                      {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
