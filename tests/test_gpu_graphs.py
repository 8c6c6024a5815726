"""Calls captured into a CUDA graph and replayed: every replay gives the oracle's result for that
replay's inputs (the schedules that tell signals apart by a per-call epoch or tag clear their
flags inside the graph), eager calls between replays still work, and a call whose scratch would
have to grow during the capture is refused instead of breaking it."""
import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import make_inputs, to_torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("algo", ["direct", "ring", "rd", "hd", "tree", "dbtree", "ll", "rd_ll", "tree_ll",
                                  "dbtree_ll"])
def test_allreduce_graph_replays(algo):
    p, n = 8, 3 * 4096 + 40  # int32: exact, so every schedule matches the plain sum bit for bit
    c = SC.SimComm(p)
    try:
        x = [torch.zeros(n, dtype=torch.int32, device="cuda") for _ in range(p)]
        y = [torch.zeros(n, dtype=torch.int32, device="cuda") for _ in range(p)]
        c.allreduce(x, y, op="sum", algo=algo)  # sizes the scratch outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            c.allreduce(x, y, op="sum", algo=algo)
        for it in range(4):
            ins = make_inputs("int24", p, n, "int32", f"graph.{algo}.{it}")
            for r in range(p):
                x[r].copy_(to_torch(ins[r], "int32"))
            g.replay()
            if it == 1:  # an eager call between replays, on other buffers
                z = [torch.empty_like(t) for t in x]
                c.allreduce(x, z, op="sum", algo=algo)
                torch.cuda.synchronize()
                assert torch.equal(z[0], z[p - 1])
            torch.cuda.synchronize()
            assert c.async_error() == SC.OK
            want = O.allreduce(ins, "int32", "sum")
            for r in range(p):
                np.testing.assert_array_equal(y[r].cpu().numpy(), want[r], err_msg=f"replay {it} rank {r}")
        del g
    finally:
        c.close()


@pytest.mark.parametrize("coll", ["reduce_scatter", "allgather", "alltoall", "broadcast", "reduce"])
def test_ring_variants_graph_replays(coll):
    p, n = 4, 4 * 9000
    m = n // p
    c = SC.SimComm(p)
    try:
        x = [torch.zeros(n, dtype=torch.int32, device="cuda") for _ in range(p)]
        y = [torch.zeros(n, dtype=torch.int32, device="cuda") for _ in range(p)]

        def call():
            if coll == "reduce_scatter":
                c.reduce_scatter(x, [t[:m] for t in y], algo="ring")
            elif coll == "allgather":
                c.allgather([t[:m] for t in x], y, algo="ring")
            elif coll == "alltoall":
                c.alltoall(x, y, algo="ring")
            elif coll == "broadcast":
                c.broadcast(x, y, 1, algo="ring")
            else:
                c.reduce(x, y, 2, algo="ring")

        call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        for it in range(3):
            ins = make_inputs("int24", p, n, "int32", f"graph.{coll}.{it}")
            for r in range(p):
                x[r].copy_(to_torch(ins[r], "int32"))
            g.replay()
            torch.cuda.synchronize()
            assert c.async_error() == SC.OK
            if coll == "reduce_scatter":
                want = O.reduce_scatter(ins, "int32", "sum")
                got = [t[:m].cpu().numpy() for t in y]
            elif coll == "allgather":
                want = O.allgather([a[:m] for a in ins], "int32")
                got = [t.cpu().numpy() for t in y]
            elif coll == "alltoall":
                want = O.alltoall(ins, "int32")
                got = [t.cpu().numpy() for t in y]
            elif coll == "broadcast":
                want = [ins[1]] * p
                got = [t.cpu().numpy() for t in y]
            else:
                want = [O.reduce(ins, "int32", "sum", 2)]
                got = [y[2].cpu().numpy()]
            for w, h in zip(want, got):
                np.testing.assert_array_equal(h, w)
        del g
    finally:
        c.close()


def test_scratch_growth_is_refused_under_capture():
    p, n = 4, 1 << 16
    c = SC.SimComm(p)
    try:
        x = [torch.ones(n, device="cuda") for _ in range(p)]
        y = [torch.empty(n, device="cuda") for _ in range(p)]
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with pytest.raises(SC.SimCommError) as e:
            with torch.cuda.graph(g, stream=s):
                c.allreduce(x, y, algo="ring")  # first ring call: its flags and partials do not exist yet
        assert e.value.status == SC.UNSUPPORTED
        del g
        torch.cuda.synchronize()
        c.allreduce(x, y, algo="ring")  # the communicator still works eagerly
        torch.cuda.synchronize()
        assert torch.equal(y[0], torch.full_like(y[0], float(p)))
    finally:
        c.close()


@pytest.mark.parametrize("algo", ["ring", "tree", "ll"])
def test_graph_replays_after_the_scratch_grew(algo):
    """An eager call larger than the captured one grows the communicator's scratch; the graph still
    holds the old buffers, which stay allocated, so its replays stay correct."""
    p, n_small, n_big = 4, 4 * 3001, 4 * 60001
    c = SC.SimComm(p)
    try:
        x = [torch.zeros(n_small, dtype=torch.int32, device="cuda") for _ in range(p)]
        y = [torch.zeros(n_small, dtype=torch.int32, device="cuda") for _ in range(p)]
        c.allreduce(x, y, algo=algo)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            c.allreduce(x, y, algo=algo)
        big_in = make_inputs("int24", p, n_big, "int32", f"graph.grow.{algo}")
        bx = [to_torch(a, "int32") for a in big_in]
        by = [torch.empty_like(t) for t in bx]
        c.allreduce(bx, by, algo=algo)  # grows the flags / partials / slots
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        np.testing.assert_array_equal(by[1].cpu().numpy(), O.allreduce(big_in, "int32", "sum")[1])
        for it in range(2):
            ins = make_inputs("int24", p, n_small, "int32", f"graph.grow.{algo}.{it}")
            for r in range(p):
                x[r].copy_(to_torch(ins[r], "int32"))
            g.replay()
            torch.cuda.synchronize()
            assert c.async_error() == SC.OK
            want = O.allreduce(ins, "int32", "sum")
            for r in range(p):
                np.testing.assert_array_equal(y[r].cpu().numpy(), want[r])
        del g
    finally:
        c.close()
