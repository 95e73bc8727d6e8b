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
        # the end-to-end leg: same reduction, and the bytes of every rank
        e2e = bench.e2e_record(ops, 50, [0.030, 0.020][rank], world, torch.device("cpu"),
                               25165824, 25165824)
        q.put((rank, t_max, bench.whole_job_tops(ops, steps, world, t_max), e2e))
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
    res = sorted((q.get(timeout=10) for _ in range(2)), key=lambda r: r[0])
    assert res[0][1] == res[1][1] == 0.025
    expected = 2 * 2 * 4096 * 12288 * 3072 * 100 * 2 / 0.025 / 1e12
    assert res[0][2] == pytest.approx(expected)
    e0, e1 = res[0][3], res[1][3]
    assert e0 == e1                                    # every rank agrees
    assert e0["ms_per_step"] == pytest.approx(0.030 / 50 * 1e3)   # the slowest rank
    assert e0["value"] == pytest.approx(2 * 2 * 4096 * 12288 * 3072 * 50 * 2 / 0.030 / 1e12,
                                        rel=1e-3)
    assert e0["h2d_bytes_per_step"] == e0["d2h_bytes_per_step"] == 2 * 25165824


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1, None) == 0.5
