"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): the job's
time is the max over ranks and its throughput counts every rank's replica.
The decode path itself has no exchange step, so replicas need no collective
beyond this timing reduction."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = bench.max_over_ranks(1.0 + rank * 0.5, world)   # rank 1 is slower
        v = bench.job_tokens_per_s(16, world, t)
        bench.barrier(world)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in got:
        assert t == pytest.approx(1.5)                    # the slowest rank's time
        assert v == pytest.approx(16 * 2 / 1.5e-3)        # both replicas' sequences count


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.job_tokens_per_s(16, 1, 1.0) == pytest.approx(16000.0)
