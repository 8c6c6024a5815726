"""GPU parity of the ring AllReduce on the low-latency protocol: the same schedule and rounding as
the ring path, so it must equal the oracle's ring emulation bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import Guarded, make_inputs

pytestmark = pytest.mark.gpu

_C = {}


def comm(p):
    if p not in _C:
        _C[p] = SC.SimComm(p)
    return _C[p]


@pytest.mark.parametrize("p", [2, 3, 4, 5, 8, 16, 64])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("op", ["sum", "min", "max", "avg"])
def test_ll_allreduce_parity(p, dtype, op):
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    for n in (1, 2, 7, 100, 4099, 70001):
        ins = make_inputs("int24" if dtype == "int32" else "normal", p, n, dtype, f"ll.{p}.{n}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(n, dtype) for _ in ins]
        for _ in range(2):  # a second call reuses the slots under new tags
            c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo="ll")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = O.ring_allreduce(ins, dtype, op)
        for r in range(p):
            assert out[r].guards_intact() and src[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"n={n} r={r}")
            np.testing.assert_array_equal(src[r].numpy(), ins[r])


def test_ll_in_place_unaligned_and_worked_example():
    c = comm(4)
    ins = [np.array(v, np.float32) for v in ([1, 2], [3, 4], [0, 1], [6, 7])]
    src = [Guarded(2, "fp32", fill=x) for x in ins]
    out = [Guarded(2, "fp32") for _ in ins]
    c.allreduce([b.t for b in src], [b.t for b in out], op="sum", algo="ll")
    torch.cuda.synchronize()
    for b in out:
        assert list(b.numpy()) == [10.0, 14.0]
    n = 4 * 1003 + 3
    xs = make_inputs("normal", 4, n, "bf16", "ll.ip", sigma=1.0)
    want = O.ring_allreduce(xs, "bf16", "avg")
    buf = [Guarded(n, "bf16", offset=1, fill=x) for x in xs]
    c.allreduce([b.t for b in buf], [b.t for b in buf], op="avg", algo="ll")
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(4):
        np.testing.assert_array_equal(buf[r].numpy(), want[r])


def test_ll_limits():
    c = comm(8)
    big = [torch.zeros(8 << 20, device="cuda") for _ in range(8)]  # 8 * 13 * 1 Mi * 8 B > 256 MiB
    with pytest.raises(SC.SimCommError) as e:
        c.allreduce(big, big, algo="ll")
    assert e.value.status == SC.UNSUPPORTED
    t = [torch.ones(64, device="cuda") for _ in range(8)]
    u = [torch.zeros(64, device="cuda") for _ in range(8)]
    with pytest.raises(SC.SimCommError) as e:  # the LL ring serves AllReduce, ReduceScatter, AllGather
        c.alltoall(t, u, algo="ll")
    assert e.value.status == SC.UNSUPPORTED


@pytest.mark.parametrize("p", [2, 4, 8, 16, 64])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("op", ["sum", "min", "max", "avg"])
def test_rd_ll_allreduce_parity(p, dtype, op):
    """Recursive doubling on the LL protocol: the same arithmetic as the butterfly executor's
    recursive doubling, so it must equal the oracle's recursive-doubling emulation bit for bit."""
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    for n in (1, 7, 100, 4099, 18001) if p <= 16 else (1, 7, 100, 4099):
        ins = make_inputs("int24" if dtype == "int32" else "normal", p, n, dtype, f"rdll.{p}.{n}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(n, dtype) for _ in ins]
        for _ in range(2):
            c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo="rd_ll")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = O.rd_allreduce(ins, dtype, op)
        for r in range(p):
            assert out[r].guards_intact() and src[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"n={n} r={r}")


def test_rd_ll_in_place_and_limits():
    c = comm(8)
    n = 8 * 1001
    xs = make_inputs("normal", 8, n, "bf16", "rdll.ip", sigma=1.0)
    want = O.rd_allreduce(xs, "bf16", "avg")
    buf = [Guarded(n, "bf16", offset=1, fill=x) for x in xs]
    c.allreduce([b.t for b in buf], [b.t for b in buf], op="avg", algo="rd_ll")
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(8):
        np.testing.assert_array_equal(buf[r].numpy(), want[r])
    big = [torch.zeros(4 << 20, device="cuda") for _ in range(8)]  # more than 8 elements per thread
    with pytest.raises(SC.SimCommError) as e:
        c.allreduce(big, big, algo="rd_ll")
    assert e.value.status == SC.UNSUPPORTED
    c3 = SC.SimComm(3)
    t = [torch.ones(16, device="cuda") for _ in range(3)]
    with pytest.raises(SC.SimCommError) as e:
        c3.allreduce(t, t, algo="rd_ll")
    assert e.value.status == SC.UNSUPPORTED
    c3.close()


@pytest.mark.parametrize("p", [2, 3, 5, 8, 16, 64])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("op", ["sum", "min", "avg"])
def test_ll_reduce_scatter_parity(p, dtype, op):
    """The ring ReduceScatter on the LL protocol equals the oracle's ring reduce-scatter emulation."""
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    for m in (1, 3, 257, 4099):
        n = m * p
        ins = make_inputs("int24" if dtype == "int32" else "normal", p, n, dtype, f"llrs.{p}.{m}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(m, dtype) for _ in ins]
        c.reduce_scatter([b.t for b in src], [b.t for b in out], op=op, algo="ll")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = O.ring_reduce_scatter(ins, dtype, op)
        for r in range(p):
            assert out[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"m={m} r={r}")


@pytest.mark.parametrize("p", [2, 3, 5, 8, 16, 64])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
def test_ll_allgather_parity(p, dtype):
    """The ring AllGather on the LL protocol equals the oracle's ring all-gather (and AllGather's layout)."""
    c = comm(p)
    for m in (1, 3, 257, 4099):
        n = m * p
        shards = make_inputs("int24" if dtype == "int32" else "normal", p, m, dtype, f"llag.{p}.{m}")
        src = [Guarded(m, dtype, fill=x) for x in shards]
        out = [Guarded(n, dtype) for _ in shards]
        c.allgather([b.t for b in src], [b.t for b in out], algo="ll")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = O.ring_allgather(shards, dtype)
        for r in range(p):
            assert out[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"m={m} r={r}")


def test_ll_reduce_scatter_and_allgather_in_place():
    p, m = 4, 1001
    n = p * m
    c = comm(p)
    xs = make_inputs("normal", p, n, "fp32", "llip.rs", sigma=1.0)
    want = O.ring_reduce_scatter(xs, "fp32", "sum")
    full = [Guarded(n, "fp32", fill=x) for x in xs]
    c.reduce_scatter([b.t for b in full], [b.t[r * m:(r + 1) * m] for r, b in enumerate(full)], op="sum", algo="ll")
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(p):
        np.testing.assert_array_equal(full[r].numpy()[r * m:(r + 1) * m], want[r])
    shards = make_inputs("normal", p, m, "bf16", "llip.ag", sigma=1.0)
    want = O.ring_allgather(shards, "bf16")
    bufs = [Guarded(n, "bf16") for _ in range(p)]
    for r in range(p):
        bufs[r].t[r * m:(r + 1) * m].copy_(torch.from_numpy(shards[r].view(np.int16)).view(torch.bfloat16).cuda())
    c.allgather([b.t[r * m:(r + 1) * m] for r, b in enumerate(bufs)], [b.t for b in bufs], algo="ll")
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(p):
        np.testing.assert_array_equal(bufs[r].numpy(), want[r])


@pytest.mark.parametrize("p", [2, 3, 5, 8, 13, 16, 63, 64])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("op", ["sum", "max", "avg"])
@pytest.mark.parametrize("algo", ["tree_ll", "dbtree_ll"])
def test_tree_ll_allreduce_parity(p, dtype, op, algo):
    """The single and double binary trees on the LL protocol equal the oracle's tree folds bit for
    bit."""
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    for n in (1, 2, 3, 7, 100, 4099) + ((70001,) if p <= 16 else ()):
        ins = make_inputs("int24" if dtype == "int32" else "normal", p, n, dtype, f"trll.{p}.{n}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(n, dtype) for _ in ins]
        for _ in range(2):
            c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = O.tree_allreduce(ins, dtype, op, double_tree=(algo == "dbtree_ll"))
        for r in range(p):
            assert out[r].guards_intact() and src[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"n={n} r={r}")


@pytest.mark.parametrize("algo", ["tree_ll", "dbtree_ll"])
def test_tree_ll_in_place(algo):
    c = comm(5)
    n = 5 * 1001 + 2
    xs = make_inputs("normal", 5, n, "bf16", "trll.ip", sigma=1.0)
    want = O.tree_allreduce(xs, "bf16", "avg", double_tree=(algo == "dbtree_ll"))
    buf = [Guarded(n, "bf16", offset=1, fill=x) for x in xs]
    c.allreduce([b.t for b in buf], [b.t for b in buf], op="avg", algo=algo)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(5):
        np.testing.assert_array_equal(buf[r].numpy(), want[r])
