"""The replica path with more than one rank (one process per GPU in the bench):
every timed figure is the max over ranks, the whole-job rate counts every
rank's tokens over the slowest rank's time, the ranks take the same collective
steps in the same order, and only rank 0 runs the reference arm.  Run here as
two gloo ranks on the CPU."""
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    r = bench.Ranks(dist, "cpu")
    r.barrier()
    # rank-dependent timings: rank 1 is the slowest for the first, rank 0 for the second
    a, b = r.max(10.0 + rank, 20.0 - rank)
    single = r.max(3.0 * (rank + 1))
    rate = r.rate(units_per_rank=100, max_ms=a)
    # the reference arm: only rank 0 does any work
    class Args:
        steps, warmup = 1, 0
    ref_rc = bench.run_reference(Args, rank, world) if rank != 0 else None
    w = r.world
    r.barrier()
    dist.destroy_process_group()
    q.put((rank, a, b, single, rate, w, ref_rc))


def test_two_gloo_ranks_max_and_rate():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(k, 2, port, q)) for k in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, a, b, single, rate, world, ref_rc in out:
        assert (a, b) == (11.0, 20.0)          # max over ranks, element by element
        assert single == 6.0
        assert world == 2
        assert rate == pytest.approx(2 * 100 / 11e-3)
        if rank == 1:
            assert ref_rc == 0                   # the other ranks exit without work


def test_single_rank_has_no_collectives():
    import bench
    r = bench.Ranks()
    assert r.world == 1
    assert r.max(4.0) == 4.0 and r.max(1.0, 2.0) == [1.0, 2.0]
    assert r.rate(5, 10.0) == pytest.approx(500.0)
    r.barrier()
