"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, max time and summed units."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    t, u = bench.aggregate(10.0 * (rank + 1), 100.0 + rank, world, device="cpu")
    q.put((rank, t, u))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregate_takes_max_time_and_sums_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, t, u in res:
        assert t == pytest.approx(20.0) and u == pytest.approx(201.0)


def test_single_rank_aggregate_is_identity():
    import bench

    assert bench.aggregate(3.5, 7.0, 1) == (3.5, 7.0)
