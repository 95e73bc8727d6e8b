"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): ranks
agree on the max elapsed time, barriers line up, and rank 0 alone reports;
no data-path collective is involved (replicas)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [0.010, 0.025][rank]
        dist.barrier()
        t = torch.tensor([elapsed], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.barrier()
        ops, steps = 2 * 512 * 4096 * 4096, 100
        value = ops * steps * world / float(t.item()) / 1e12
        q.put((rank, float(t.item()), value))
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
    expected = 2 * 512 * 4096 * 4096 * 100 * 2 / 0.025 / 1e12
    assert res[0][2] == pytest.approx(expected)
