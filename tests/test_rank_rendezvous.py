"""Host side of the rank views on CPU: two gloo ranks exchange buffer handles in rank order, and each
builds its rank-ordered pointer list (its own pointer, the peers' mapped through the opener)."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from collective_communication_primitives_b200 import ranks
    handle = bytes([rank]) * 64
    got = ranks.exchange(handle)
    opened = []
    ptrs = ranks.open_handles(got, rank, 1000 + rank, lambda h: opened.append(h) or 5000 + h[0])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, [g[0] for g in got], ptrs, [h[0] for h in opened]))


def test_handles_are_exchanged_in_rank_order():
    world, port = 3, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, order, ptrs, opened in res:
        assert order == [0, 1, 2]                    # every rank sees every handle, in rank order
        assert ptrs[rank] == 1000 + rank             # its own buffer is used directly
        assert [ptrs[q] for q in range(world) if q != rank] == [5000 + q for q in range(world) if q != rank]
        assert opened == [q for q in range(world) if q != rank]  # only the peers' handles are opened
