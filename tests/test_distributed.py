"""Multi-process plumbing of bench.py on CPU: gloo, world size 2.

The path does not shard (batch-1 decode; every rank is an independent replica),
so the only cross-rank steps are the timing reduction (max over ranks), the
whole-job rate, and the rule that the reference arm runs on rank 0 alone.
"""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        ms = 10.0 + 5.0 * rank  # rank 1 is the slow replica
        m = bench.max_over_ranks(ms, dist, "cpu")
        rate = bench.whole_job_rate(100, world, m)

        class Args:
            steps, warmup = 1, 0

        ref = bench.run_reference(Args, rank, world) if rank != 0 else "rank 0 not run here"
        q.put((rank, m, rate, ref))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timing_is_max_over_ranks_and_rate_counts_every_rank():
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r[0] for r in results] == [0, 1]
    for rank, m, rate, _ in results:
        assert m == 15.0  # every rank sees the slowest replica's time
        assert rate == pytest.approx(100 * 2 / 0.015)  # units of both ranks over that time
    assert results[1][3] is None  # the reference arm does no work on rank 1
    assert all(p.exitcode == 0 for p in procs)


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(12.5, None, "cpu") == 12.5
    assert bench.whole_job_rate(3328, 1, 67.87) == pytest.approx(3328 / 0.06787)
