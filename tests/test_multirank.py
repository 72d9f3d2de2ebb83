"""World-size-2 gloo checks of the benchmark's multi-rank host logic (CPU):
the max-over-ranks timing reduction and the barrier, as bench.py uses them
under torchrun (one process per GPU, weak scaling, no data-path collective)."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        bench.barrier(ws)
        t = bench.max_over_ranks(1.5 + rank, ws)  # rank 1 is the slow one
        q.put((r, ws, local, t))
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2, 0, 2.5), (1, 2, 1, 2.5)]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_step_bytes_accounting():
    import bench
    b = bench.step_bytes(1024, 131072)
    n = 1024 * 131072
    assert b["mx_quantize"] == n * (2 + 0.5 + 1 / 32)
    assert b["nv_quantize"] == n * (4 + 0.5 + 1 / 16)
    assert abs(sum(b.values()) / n - (2.53125 + 4.5625 + 2.53125 + 2.5625)) < 1e-12
