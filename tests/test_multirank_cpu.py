"""bench.py's multi-rank plumbing on CPU: two gloo ranks, barrier, max over ranks, weak-scaling
aggregation, and rank 0 alone reporting (no GPU; ranks are spawned processes)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = bench.Ranks(dist, torch.device("cpu"))
        assert (r.rank, r.world) == (rank, world)
        r.barrier()
        # each rank "timed" a different duration and token count per step
        my_ms = 100.0 + 50.0 * rank
        my_dec = 80.0 + 10.0 * rank
        t_max, dec_max = r.max(my_ms, my_dec)
        tokens = 8193 * 10
        value = bench.weak_scaling_value(world, tokens, 64, t_max)
        q.put((rank, t_max, dec_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_weak_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t_max, dec_max, value in got:
        assert t_max == 150.0 and dec_max == 90.0
        assert value == pytest.approx(2 * 8193 * 10 * 64 / 0.150)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks()
    r.barrier()
    assert r.max(3.0) == 3.0 and r.max(1.0, 2.0) == (1.0, 2.0)
    assert bench.weak_scaling_value(1, 100, 64, 1000.0) == 6400.0
