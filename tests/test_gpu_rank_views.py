"""Rank views on one GPU: every rank is its own process with its own CUDA context; buffers are
allocated by the library (sim_ipc_alloc), their handles exchanged over gloo and mapped into the
other processes (sim_ipc_open), and each rank's collective reads its peers' buffers directly. Each
rank's output is compared bit for bit with the oracle (every rank regenerates every rank's seeded
inputs). No kernel waits on another process: the ranks meet only at host barriers between calls.
A rank that leaves between calls makes the others' next call fail on the host with
COLL_ERR_TIMEOUT."""
import os
import socket

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _setup(rank, world, port, timeout_s):
    import sys
    from datetime import timedelta

    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=timeout_s))
    torch.cuda.set_device(0)


def _bits(a):
    import numpy as np
    return a.view(np.uint32) if a.dtype == np.float32 else a


def _collectives(rank, world, port, dtype, op, q):
    try:
        _setup(rank, world, port, 60)
        import numpy as np
        import torch.distributed as dist

        import oracle as O
        from collective_communication_primitives_b200 import ranks
        from gpu_helpers import make_inputs, to_numpy, to_torch
        p, m = world, 4099
        n = p * m
        d = ranks.BYTES[dtype]
        kind = "int24" if dtype == "int32" else "normal"
        ins = make_inputs(kind, p, n, dtype, f"ranks.{p}.{dtype}")
        comm = ranks.RankComm()
        sbuf, rbuf = ranks.SharedBuffer(n * d), ranks.SharedBuffer(n * d)
        sbuf.view(dtype, n).copy_(to_torch(ins[rank], dtype))
        sends = comm.register(sbuf)
        out = rbuf.view(dtype, n)
        sentinel = to_torch(np.full(n, 7, {"int32": np.int32, "fp32": np.float32, "bf16": np.uint16}[dtype]), dtype)

        def got(count):
            return to_numpy(out[:count], dtype)

        def check(name, want):
            w = np.asarray(want)
            g = got(w.size)
            assert np.array_equal(_bits(g), _bits(w)), f"{name}: rank {rank} differs"

        acc = "exact" if (dtype == "int32" or op in ("min", "max")) else "rankfold"
        comm.allreduce(sends, rbuf.ptr, n, dtype, op=op)
        check("allreduce", O.allreduce(ins, dtype, op, acc=acc)[rank])
        comm.reduce_scatter(sends, rbuf.ptr, n, dtype, op=op)
        check("reduce_scatter", O.reduce_scatter(ins, dtype, op, acc=acc)[rank])
        comm.alltoall(sends, rbuf.ptr, n, dtype)
        check("alltoall", O.alltoall(ins, dtype)[rank])
        root = p - 1
        comm.broadcast(sends, rbuf.ptr, root, n, dtype)
        check("broadcast", O.broadcast(ins[root], p, dtype, root)[rank])
        comm.scatter(sends, rbuf.ptr, root, n, dtype)
        check("scatter", O.scatter(ins[root], p, dtype, root)[rank])
        out.copy_(sentinel)
        comm.reduce(sends, rbuf.ptr, root, n, dtype, op=op)
        if rank == root:
            check("reduce", O.reduce(ins, dtype, op, root, acc=acc))
        else:
            check("reduce leaves non-roots untouched", to_numpy(sentinel, dtype))
        # AllGather / Gather of the first m elements of every rank's input
        shards = [x[:m] for x in ins]
        comm.allgather(sends, rbuf.ptr, n, dtype)
        check("allgather", O.allgather(shards, dtype)[rank])
        out.copy_(sentinel)
        comm.gather(sends, rbuf.ptr, 0, n, dtype)
        check("gather", O.gather(shards, dtype, 0) if rank == 0 else to_numpy(sentinel, dtype))
        # All-to-Allv on a seeded count matrix, the same on every rank; rank i sends the first
        # Σ_j c[i][j] elements of its input
        import torch

        from collective_communication_primitives_b200 import synth as S
        cmat = S.ints(f"ranks.counts.{p}", p * p, 0, m // p).astype(np.int64).reshape(p, p)
        counts_dev = torch.from_numpy(cmat).cuda()
        send_cap = [n] * p
        recv_cap = [int(cmat[:, j].sum()) for j in range(p)]
        comm.alltoallv(sends, rbuf.ptr, counts_dev, send_cap, recv_cap, dtype)
        want_v, _ = O.alltoallv([ins[i][:int(cmat[i].sum())] for i in range(p)], cmat, dtype)
        check("alltoallv", want_v[rank])
        assert comm.async_error() == 0
        comm.sync()
        comm.close()  # every mapping closed before any owner frees its buffers
        dist.barrier()
        sbuf.close()
        rbuf.close()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent
        import traceback
        q.put((rank, f"{type(e).__name__}: {e}\n{traceback.format_exc()}"))


def _spawn(target, world, *args, timeout=300):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=timeout) for _ in range(world))
    for pr in procs:
        pr.join(timeout=120)
    return res, [pr.exitcode for pr in procs]


@pytest.mark.parametrize("world,dtype,op", [(2, "fp32", "sum"), (3, "bf16", "avg"), (4, "int32", "sum"),
                                            (4, "fp32", "max")])
def test_rank_views_match_the_oracle(world, dtype, op):
    res, codes = _spawn(_collectives, world, dtype, op)
    assert all(v == "ok" for v in res.values()), res
    assert codes == [0] * world


def _report_and_exit(q, item):
    """Puts the result and flushes the queue's feeder thread before leaving without cleanup (the
    process group is broken, so no orderly shutdown)."""
    q.put(item)
    q.close()
    q.join_thread()
    os._exit(0)


def _leaver(rank, world, port, q):
    try:
        _setup(rank, world, port, 5)
        from collective_communication_primitives_b200 import ranks
        from collective_communication_primitives_b200 import simcomm as SC
        n = 2 * 1024
        comm = ranks.RankComm()
        sbuf, rbuf = ranks.SharedBuffer(n * 4), ranks.SharedBuffer(n * 4)
        sbuf.view("fp32", n).fill_(1.0)
        sends = comm.register(sbuf)
        comm.allreduce(sends, rbuf.ptr, n, "fp32")  # both ranks take part once
        if rank == 1:  # leaves between calls, with nothing of its own in flight
            comm.close()
            _report_and_exit(q, (rank, "left"))
        try:
            comm.allreduce(sends, rbuf.ptr, n, "fp32")
            _report_and_exit(q, (rank, "no error"))
        except SC.SimCommError as e:
            _report_and_exit(q, (rank, "timeout" if e.status == SC.TIMEOUT else f"status {e.status}"))
    except Exception as e:
        _report_and_exit(q, (rank, f"{type(e).__name__}: {e}"))


def test_a_rank_that_leaves_makes_the_next_call_time_out():
    res, _ = _spawn(_leaver, 2, timeout=180)
    assert res == {0: "timeout", 1: "left"}, res


def _forms(rank, world, port, q):
    """The in-place forms a rank view accepts (the root's own Broadcast and Scatter), the ones it
    refuses (an output over an input a peer may still read), and the schedules it does not run."""
    try:
        _setup(rank, world, port, 60)
        import numpy as np
        import torch.distributed as dist

        import oracle as O
        from collective_communication_primitives_b200 import ranks
        from collective_communication_primitives_b200 import simcomm as SC
        from gpu_helpers import make_inputs, to_numpy, to_torch
        p, m = world, 1031
        n = p * m
        ins = make_inputs("normal", p, n, "fp32", "ranks.forms")
        comm = ranks.RankComm()
        buf = ranks.SharedBuffer(n * 4)
        buf.view("fp32", n).copy_(to_torch(ins[rank], "fp32"))
        sends = comm.register(buf)
        root = 1
        out = ranks.SharedBuffer(n * 4)
        # the root broadcasts in place (its output is its input); the others receive into their own
        recv = buf.ptr if rank == root else out.ptr
        comm.broadcast(sends, recv, root, n, "fp32")
        got = to_numpy((buf if rank == root else out).view("fp32", n), "fp32")
        assert np.array_equal(got.view(np.uint32), ins[root].view(np.uint32)), "broadcast"
        # the root scatters in place: its block stays where it is
        recv = buf.ptr + rank * m * 4 if rank == root else out.ptr
        comm.scatter(sends, recv, root, n, "fp32")
        got = to_numpy((buf.view("fp32", m, offset=rank * m) if rank == root else out.view("fp32", m)), "fp32")
        want = O.scatter(ins[root], p, "fp32", root)[rank]
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), "scatter"
        # refused, on every rank alike: an in-place AllReduce (peers still read the input) and a
        # ring schedule
        codes = []
        for call in (lambda: comm.allreduce(sends, buf.ptr, n, "fp32"),
                     lambda: comm.allreduce(sends, out.ptr, n, "fp32", algo="ring")):
            try:
                call()
                codes.append(0)
            except SC.SimCommError as e:
                codes.append(e.status)
        assert codes == [SC.INVALID_ARG, SC.UNSUPPORTED], codes
        comm.sync()
        comm.close()
        dist.barrier()
        buf.close()
        out.close()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as e:
        import traceback
        q.put((rank, f"{type(e).__name__}: {e}\n{traceback.format_exc()}"))


def test_rank_view_forms_and_refusals():
    res, codes = _spawn(_forms, 3)
    assert all(v == "ok" for v in res.values()), res
    assert codes == [0, 0, 0]


def _moe(rank, world, port, dtype, T, q):
    """The MoE dispatch and combine as rank views: each rank's dispatch reads every rank's token rows
    and expert ids where they lie (IPC mappings) and writes only its own receive rows and routing
    map; its combine reads the expert-output rows of every rank at its own tokens' routes. Both are
    compared bit for bit with the oracle's result for this rank."""
    try:
        _setup(rank, world, port, 60)
        import numpy as np
        import torch
        import torch.distributed as dist

        import oracle as O
        from collective_communication_primitives_b200 import ranks
        from collective_communication_primitives_b200 import simcomm as SC
        from collective_communication_primitives_b200 import synth as S
        from gpu_helpers import to_numpy, to_torch
        p = world
        k, E, H = 2, 4 * p, 40
        d = ranks.BYTES[dtype]
        ids = S.moe_routes(p, T, E, k, 1.1, 5 + p)
        xs = [S.normal(f"ranks.moe.x.{i}", T * H, 1.0, dtype).reshape(T, H) for i in range(p)]
        ref = O.moe_dispatch(xs, list(ids), E, p * T * k, dtype)
        cap = int(ref["recv_counts"].max())
        comm = ranks.RankComm()
        xbuf, ibuf, ybuf = ranks.SharedBuffer(T * H * d), ranks.SharedBuffer(T * k * 4), ranks.SharedBuffer(cap * H * d)
        xbuf.view(dtype, T * H).copy_(to_torch(xs[rank].ravel(), dtype))
        ibuf.view("int32", T * k).copy_(torch.from_numpy(np.ascontiguousarray(ids[rank].ravel(), dtype=np.int32)))
        xp, ip, yp = comm.register(xbuf), comm.register(ibuf), comm.register(ybuf)
        pos = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        ec = torch.full((p, E), -1, dtype=torch.int64, device="cuda")
        rc = torch.full((p,), -1, dtype=torch.int64, device="cuda")
        comm.moe_dispatch(xp, ip, E, ybuf.ptr, T, k, H, dtype, cap, route_pos=pos.data_ptr(), expert_counts=ec,
                          recv_counts=rc)
        assert np.array_equal(rc.cpu().numpy(), ref["recv_counts"]), "recv_counts"
        assert np.array_equal(ec.cpu().numpy(), ref["expert_counts"]), "expert_counts"
        assert np.array_equal(pos.cpu().numpy(), ref["pos"][rank]), "route_pos"
        nr = int(ref["recv_counts"][rank])
        got = to_numpy(ybuf.view(dtype, nr * H), dtype).reshape(nr, H)
        assert np.array_equal(got, ref["recv"][rank][:nr]), f"rank {rank}: received rows differ"
        # combine: the received rows stand for the experts' outputs
        ws = S.moe_gate_weights(p, T, k, 9)
        res = [S.normal(f"ranks.moe.res.{i}", T * H, 1.0, dtype).reshape(T, H) for i in range(p)]
        w_t = to_torch(ws[rank].ravel(), "fp32").view(T, k)
        res_t = to_torch(res[rank].ravel(), dtype)
        out = torch.empty_like(res_t)
        comm.moe_combine(yp, cap, ibuf.ptr, pos.data_ptr(), w_t.data_ptr(), E, out.data_ptr(), T, k, H, dtype,
                         residual=res_t.data_ptr())
        want = O.moe_combine([r[:cap] for r in ref["recv"]], list(ids), list(ws), dtype, E, residual=res,
                             acc="slotfold")[rank]
        assert np.array_equal(to_numpy(out, dtype).reshape(T, H), want), f"rank {rank}: combine differs"
        # the three-kernel dispatch is not built for rank views: refused on every rank, in step
        comm.set_option("moe_fused", 0)
        try:
            comm.moe_dispatch(xp, ip, E, ybuf.ptr, T, k, H, dtype, cap)
            raise AssertionError("the three-kernel dispatch ran on a rank view")
        except SC.SimCommError as e:
            assert e.status == SC.UNSUPPORTED, e.status
        assert comm.async_error() == 0
        comm.sync()
        comm.close()
        dist.barrier()
        for b in (xbuf, ibuf, ybuf):
            b.close()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent
        import traceback
        q.put((rank, f"{type(e).__name__}: {e}\n{traceback.format_exc()}"))


@pytest.mark.parametrize("world,dtype,T", [(2, "bf16", 700), (3, "fp32", 700), (4, "bf16", 700),
                                           (2, "fp32", 9000)])  # 6 counting tiles per rank; 71 (long path)
def test_rank_view_moe_dispatch_and_combine_match_the_oracle(world, dtype, T):
    res, codes = _spawn(_moe, world, dtype, T)
    assert all(v == "ok" for v in res.values()), res
    assert codes == [0] * world
