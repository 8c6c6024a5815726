"""Failure detection of the latency schedules, tested without a GPU fault: host-side fault injection
(option fault_skip_rank: one rank never signals or sends) makes a successor's bounded wait run out,
so the call reports COLL_ERR_TIMEOUT (or COLL_ERR_ABORTED after sim_comm_abort) and the kernel
returns; sim_comm_reset makes the communicator usable again."""
import time

import numpy as np
import pytest
import torch

from collective_communication_primitives_b200 import simcomm as SC

pytestmark = pytest.mark.gpu


def run(c, kind, algo, t, u, p, n):
    if kind == "allreduce":
        c.allreduce(t, u, algo=algo)
    elif kind == "reduce_scatter":
        c.reduce_scatter(t, [x[:n // p] for x in u], algo=algo)
    else:
        c.allgather([x[:n // p] for x in t], u, algo=algo)


CASES = [("allreduce", a) for a in ("tree", "dbtree", "rd", "hd", "ll", "rd_ll", "tree_ll", "dbtree_ll")] + \
        [("reduce_scatter", "ll"), ("allgather", "ll")]


@pytest.mark.parametrize("kind,algo", CASES)
def test_timeout_when_a_rank_is_silent(kind, algo):
    p, n = 4, 4 * 4096
    c = SC.SimComm(p)
    c.set_option("chunk_bytes", 4096)
    c.set_option("timeout_ns", 100_000_000)
    c.set_option("fault_skip_rank", 1)
    t = [torch.ones(n, device="cuda") for _ in range(p)]
    u = [torch.zeros(n, device="cuda") for _ in range(p)]
    t0 = time.time()
    run(c, kind, algo, t, u, p, n)
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert c.async_error() == SC.TIMEOUT
    with pytest.raises(SC.SimCommError) as e:  # refused until reset
        run(c, kind, algo, t, u, p, n)
    assert e.value.status == SC.TIMEOUT
    c.set_option("fault_skip_rank", -1)
    c.reset()
    run(c, kind, algo, t, u, p, n)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    if kind == "allgather":
        assert torch.equal(u[2], torch.ones_like(u[2]))
    elif kind == "reduce_scatter":
        assert torch.equal(u[2][:n // p], torch.full_like(u[2][:n // p], float(p)))
    else:
        assert torch.equal(u[2], torch.full_like(u[2], float(p)))
    c.close()


@pytest.mark.parametrize("algo", ["tree", "ll", "rd_ll", "hd", "tree_ll"])
def test_abort_stops_a_waiting_schedule(algo):
    p, n = 4, 4 * 4096
    c = SC.SimComm(p)
    c.set_option("chunk_bytes", 4096)
    c.set_option("timeout_ns", 5_000_000_000)
    c.set_option("fault_skip_rank", 1)  # an inner tree position (a silent leaf would hold nobody up)
    t = [torch.ones(n, device="cuda") for _ in range(p)]
    u = [torch.zeros(n, device="cuda") for _ in range(p)]
    t0 = time.time()
    c.allreduce(t, u, algo=algo)
    time.sleep(0.05)
    c.abort()
    torch.cuda.synchronize()
    assert time.time() - t0 < 4.0
    assert c.async_error() == SC.ABORTED
    c.set_option("fault_skip_rank", -1)
    c.reset()
    c.allreduce(t, u, algo=algo)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    assert np.array_equal(u[3].cpu().numpy(), np.full(n, float(p), np.float32))
    c.close()


@pytest.mark.parametrize("mode", ["timeout", "abort"])
def test_fused_moe_dispatch_barrier_wait_is_bounded(mode):
    """The fused MoE dispatch's grid barrier: with fault_skip_rank = 1 its CTA 1 never arrives, so
    every other CTA's wait runs out (COLL_ERR_TIMEOUT) or ends on sim_comm_abort (COLL_ERR_ABORTED)
    and nothing is copied. The failed call leaves its per-(rank, expert) totals uncleared; after
    sim_comm_reset the next dispatch matches the oracle exactly."""
    import oracle

    from collective_communication_primitives_b200 import synth as S
    p, T, k, E, H = 4, 600, 2, 8, 16
    ids = S.moe_routes(p, T, E, k, 1.1, 3)
    xs = [S.normal(f"faults.moe.rank{r}", T * H, 1.0, "fp32").reshape(T, H) for r in range(p)]
    ref = oracle.moe_dispatch(xs, list(ids), E, p * T * k, "fp32")
    cap = int(ref["recv_counts"].max())
    x = [torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda() for a in xs]
    idx = [torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda() for a in ids]
    recv = [torch.zeros(cap, H, device="cuda") for _ in range(p)]
    c = SC.SimComm(p)
    c.set_option("timeout_ns", 100_000_000 if mode == "timeout" else 5_000_000_000)
    c.set_option("fault_skip_rank", 1)
    t0 = time.time()
    c.moe_dispatch(x, idx, E, recv)
    if mode == "abort":
        time.sleep(0.05)
        c.abort()
    torch.cuda.synchronize()
    assert time.time() - t0 < 4.0
    assert c.async_error() == (SC.TIMEOUT if mode == "timeout" else SC.ABORTED)
    assert all(int(torch.count_nonzero(g)) == 0 for g in recv), "a failed dispatch copied rows"
    c.set_option("fault_skip_rank", -1)
    c.reset()
    pos = [torch.empty(T, k, dtype=torch.int32, device="cuda") for _ in range(p)]
    c.moe_dispatch(x, idx, E, recv, route_pos=pos)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for j in range(p):
        n = int(ref["recv_counts"][j])
        assert np.array_equal(recv[j][:n].cpu().numpy(), ref["recv"][j][:n]), j
    for i in range(p):
        assert np.array_equal(pos[i].cpu().numpy(), ref["pos"][i]), i
    c.close()
