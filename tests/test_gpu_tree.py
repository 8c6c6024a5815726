"""GPU parity of the single and double binary tree AllReduce against the oracle's tree fold (bit for
bit) and the exact sum (within the stated bounds)."""
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


@pytest.mark.parametrize("p", [2, 3, 5, 8, 13, 16, 64])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("op", ["sum", "min", "max", "avg"])
@pytest.mark.parametrize("algo", ["tree", "dbtree"])
def test_tree_allreduce_parity(p, dtype, op, algo):
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    sizes = (1, 2, 7, 4099, 70001, 9 * 32768 + 5) if p <= 16 else (1, 7, 4099, 40003)
    for n in sizes:
        ins = make_inputs("int24" if dtype == "int32" else "normal", p, n, dtype, f"tr.{p}.{n}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(n, dtype) for _ in ins]
        c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want = O.tree_allreduce(ins, dtype, op, double_tree=(algo == "dbtree"))
        for r in range(p):
            assert out[r].guards_intact() and src[r].guards_intact()
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"n={n} r={r}")
            np.testing.assert_array_equal(src[r].numpy(), ins[r])
        if dtype != "int32" and op in ("sum", "avg") and p <= 16:
            check_sum_tolerance(out[0].numpy(), ins, dtype, op, p)


@pytest.mark.parametrize("algo", ["tree", "dbtree"])
@pytest.mark.parametrize("chunk_bytes", [4096, 65536])
def test_tree_many_chunks_in_place_and_unaligned(algo, chunk_bytes):
    """Small chunks (many pipelined chunks per tree), the in-place form, and unaligned buffers."""
    p, n = 6, 3 * 65536 + 11
    c = SC.SimComm(p)
    c.set_option("chunk_bytes", chunk_bytes)
    xs = make_inputs("normal", p, n, "fp32", f"tr.ch.{chunk_bytes}", sigma=1.0)
    want = O.tree_allreduce(xs, "fp32", "sum", double_tree=(algo == "dbtree"))
    buf = [Guarded(n, "fp32", fill=x) for x in xs]
    c.allreduce([b.t for b in buf], [b.t for b in buf], op="sum", algo=algo)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(p):
        assert buf[r].guards_intact()
        np.testing.assert_array_equal(buf[r].numpy(), want[r])
    src = [Guarded(n, "fp32", offset=1, fill=x) for x in xs]
    out = [Guarded(n, "fp32", offset=3) for _ in xs]
    c.allreduce([b.t for b in src], [b.t for b in out], op="sum", algo=algo)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for r in range(p):
        np.testing.assert_array_equal(out[r].numpy(), want[r])
    c.close()


def test_tree_worked_example_and_allreduce_only():
    c = comm(4) if 4 in _C else SC.SimComm(4)
    ins = [np.array(v, np.float32) for v in ([1, 2], [3, 4], [0, 1], [6, 7])]
    for algo in ("tree", "dbtree"):
        src = [Guarded(2, "fp32", fill=x) for x in ins]
        out = [Guarded(2, "fp32") for _ in ins]
        c.allreduce([b.t for b in src], [b.t for b in out], op="sum", algo=algo)
        torch.cuda.synchronize()
        for b in out:
            assert list(b.numpy()) == [10.0, 14.0]
        t = [torch.ones(16, device="cuda") for _ in range(4)]
        u = [torch.zeros(16, device="cuda") for _ in range(4)]
        with pytest.raises(SC.SimCommError) as e:
            c.reduce_scatter(t, [x[:4] for x in u], algo=algo)
        assert e.value.status == SC.UNSUPPORTED


@pytest.mark.parametrize("algo", ["tree", "dbtree"])
def test_tree_dp_bucket(algo):
    """p = 8, the 25 Mi-element DP bucket, fp32 AVG: bit-exact against the oracle's tree fold."""
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
    want = O.tree_allreduce(ins, "fp32", "avg", double_tree=(algo == "dbtree"))[0]
    np.testing.assert_array_equal(out[0].cpu().numpy(), want)
