"""GPU parity of the recursive-doubling and halving-doubling AllReduce ([Atlas] §2.3) against the
oracle's step-by-step emulations (bit for bit) and the exact sum (within the stated bounds)."""
import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import Guarded, check_sum_tolerance, make_inputs

pytestmark = pytest.mark.gpu

_C = {}


def comm(p):
    if p not in _C:
        _C[p] = SC.SimComm(p)
    return _C[p]


def emulation(algo):
    return O.rd_allreduce if algo == "rd" else O.hd_allreduce


@pytest.mark.parametrize("p", [2, 4, 8, 16])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("op", ["sum", "min", "max", "avg"])
@pytest.mark.parametrize("algo", ["rd", "hd"])
def test_butterfly_allreduce_parity(p, dtype, op, algo):
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    for n in (1, 7, p * 3 + 1, 4099, 70001, 40 * 32768 + 5):
        ins = make_inputs("int24" if dtype == "int32" else "normal", p, n, dtype, f"bf.{p}.{n}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(n, dtype) for _ in ins]
        c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = emulation(algo)(ins, dtype, op)
        for r in range(p):
            assert out[r].guards_intact() and src[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"n={n} r={r}")
            np.testing.assert_array_equal(src[r].numpy(), ins[r])
        if dtype != "int32" and op in ("sum", "avg"):
            check_sum_tolerance(out[0].numpy(), ins, dtype, op, p)


@pytest.mark.parametrize("algo", ["rd", "hd"])
def test_butterfly_worked_example_and_unaligned(algo):
    c = comm(4)
    ins = [np.array(v, np.float32) for v in ([1, 2], [3, 4], [0, 1], [6, 7])]
    src = [Guarded(2, "fp32", fill=x) for x in ins]
    out = [Guarded(2, "fp32") for _ in ins]
    c.allreduce([b.t for b in src], [b.t for b in out], op="sum", algo=algo)
    torch.cuda.synchronize()
    for b in out:
        assert list(b.numpy()) == [10.0, 14.0]
    n = 4 * 5003
    xs = make_inputs("normal", 4, n, "fp32", "bf.ua", sigma=1.0)
    src = [Guarded(n, "fp32", offset=1, fill=x) for x in xs]
    out = [Guarded(n, "fp32", offset=3) for _ in xs]
    c.allreduce([b.t for b in src], [b.t for b in out], op="sum", algo=algo)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    want = emulation(algo)(xs, "fp32", "sum")
    for r in range(4):
        np.testing.assert_array_equal(out[r].numpy(), want[r])


def test_butterfly_needs_a_power_of_two_and_allreduce():
    c = comm(3) if 3 in _C else SC.SimComm(3)
    t = [torch.ones(16, device="cuda") for _ in range(3)]
    u = [torch.zeros(16, device="cuda") for _ in range(3)]
    for algo in ("rd", "hd"):
        with pytest.raises(SC.SimCommError) as e:
            c.allreduce(t, u, algo=algo)
        assert e.value.status == SC.UNSUPPORTED
    c4 = comm(4)
    t = [torch.ones(16, device="cuda") for _ in range(4)]
    u = [torch.zeros(16, device="cuda") for _ in range(4)]
    with pytest.raises(SC.SimCommError) as e:
        c4.reduce_scatter(t, [x[:4] for x in u], algo="rd")
    assert e.value.status == SC.UNSUPPORTED


@pytest.mark.parametrize("algo", ["rd", "hd"])
def test_butterfly_dp_bucket(algo):
    """p = 8, the 25 Mi-element DP bucket, fp32 AVG: bit-exact against the emulation."""
    from collective_communication_primitives_b200 import synth as S
    p, n = 8, 25 << 20
    ins = [S.normal(f"dp.fp32.rank{r}", n, 1e-3, "fp32") for r in range(p)]
    src = [torch.from_numpy(x).cuda() for x in ins]
    out = [torch.empty_like(src[0]) for _ in range(p)]
    c = comm(8)
    c.allreduce(src, out, op="avg", algo=algo)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(1, p):
        assert torch.equal(out[r], out[0])
    want = emulation(algo)(ins, "fp32", "avg")[0]
    np.testing.assert_array_equal(out[0].cpu().numpy(), want)
