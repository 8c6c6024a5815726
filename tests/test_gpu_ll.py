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
    with pytest.raises(SC.SimCommError) as e:
        c.allgather([x[:8] for x in t], u, algo="ll")
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
