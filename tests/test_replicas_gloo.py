"""Host-side logic of the multi-GPU (replicas-only) bench path, run as two gloo
ranks on CPU: max-over-ranks timing and the job-level per-unit time."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank)          # ranks report 10 and 15 ms
        per_unit = bench.job_time_per_unit(t, steps=4, world=world)
        q.put((rank, t, per_unit))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]                # every rank sees the max
    assert all(abs(r[2] - 15.0 * 1e3 / 8) < 1e-9 for r in res)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_time_per_unit(2.0, 4, 1) == 500.0
