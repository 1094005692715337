"""The bench's multi-rank path on CPU: two `gloo` ranks, as torchrun would
start them, time their replicas independently and report the slowest
rank's time; the reference arm runs on rank 0 only."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        step_ms = [2.0, 5.0][rank]  # rank 1 is the slowest replica
        dist.barrier()
        slowest = bench.max_over_ranks(step_ms, world)
        value = bench.job_throughput(4096, world, slowest)
        # the reference arm: only rank 0 works and prints
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.run_reference(type("A", (), {"workload": "x", "batch": 0, "seq_len": 0,
                                                    "warmup": 3, "steps": 1, "gpus": world})(),
                                     rank) if rank != 0 else 0
        out.put((rank, slowest, value, rc, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_replica():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value, rc, printed in res:
        assert slowest == 5.0                        # max over ranks
        assert value == pytest.approx(2 * 4096 / 5e-3)  # both ranks' units / slowest time
        assert rc == 0
        assert printed == ""                         # only rank 0 prints a line
