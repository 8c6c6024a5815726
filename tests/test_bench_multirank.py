"""The bench's multi-GPU path on CPU: two gloo ranks, each timing its own replica; the job's time
is the slowest rank's and its throughput counts every rank's bytes."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 10.0 + 5.0 * rank          # rank 1 is slower
    t = bench.reduce_max(local_ms)
    value = bench.job_gbps(world, 1e9, t)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, value))


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value in res:
        assert t == 15.0                               # max over ranks
        assert value == pytest.approx(2 * 1e9 / 15e-3 / 1e9)  # both replicas' bytes, slowest time


def test_single_process_is_the_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.job_gbps(1, 2e9, 1.0) == pytest.approx(2000.0)
