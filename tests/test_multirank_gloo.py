"""The N>1 plumbing of bench.py on CPU: two gloo ranks, max-over-ranks timing,
whole-job throughput of independent replicas, and the reference arm running
on rank 0 only."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]
        dist.barrier()
        worst = bench.max_over_ranks(ms, dist, "cpu")
        results[rank] = (worst, bench.job_throughput(world, 4096, worst))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert results[0] == results[1]
    worst, value = results[0]
    assert worst == 5.0
    assert abs(value - 2 * 4096 / 5e-3) < 1e-6


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_ffn_token_b200.workloads import WORKLOADS
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup = 3, 3
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(Args(), WORKLOADS["mixtral"])
    assert rc == 0 and buf.getvalue() == ""


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, None, "cpu") == 2.5
    assert bench.job_throughput(1, 64, 2.0) == 32000.0
