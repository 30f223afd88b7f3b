"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): every rank runs its
own independent problem, the job's time is the max over ranks, and the value
is the units of all ranks over that time. No data-path collective exists."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms_local = 10.0 + 5.0 * rank            # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms_local)
    seed = bench.rank_seed(rank)
    value = bench.weak_value(32768, world, ms_max)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms_max, seed, value))


def test_two_rank_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, s0, v0), (r1, m1, s1, v1) = out
    assert m0 == m1 == 15.0                 # both ranks report the slowest rank's time
    assert s0 != s1                         # independent problems per rank
    assert v0 == v1 == pytest.approx(2 * 32768 / 15e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.weak_value(100, 1, 1.0) == pytest.approx(1e5)
