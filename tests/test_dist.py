"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2), driving
bench.py's own rank reduction: every rank takes part in the max-over-ranks
all-reduce, all ranks agree on the slowest rank's time, and the whole-job
value counts every rank's steps over that time.  No data-path collective is
involved (replicas)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [0.010, 0.025][rank]
        dist.barrier()
        t_max = bench.max_over_ranks(elapsed, world, torch.device("cpu"))
        dist.barrier()
        ops, steps = 2 * 2 * 4096 * 12288 * 3072, 100
        q.put((rank, t_max, bench.whole_job_tops(ops, steps, world, t_max)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] == res[1][1] == 0.025
    expected = 2 * 2 * 4096 * 12288 * 3072 * 100 * 2 / 0.025 / 1e12
    assert res[0][2] == pytest.approx(expected)


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1, None) == 0.5
