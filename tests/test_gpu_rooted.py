"""GPU parity of Scatter and Gather ([Eight] §3.3, §4.3) against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import Guarded, make_inputs, to_torch

pytestmark = pytest.mark.gpu

_C = {}


def comm(p):
    if p not in _C:
        _C[p] = SC.SimComm(p)
    return _C[p]


def as_dtype(x, dtype):
    return x.view(np.float32).copy() if dtype == "fp32" else (x.astype(np.uint16) if dtype == "bf16" else x)


@pytest.mark.parametrize("p", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("dtype", ["int32", "fp32", "bf16"])
@pytest.mark.parametrize("variant", [-1, 0, 5])
def test_scatter_gather_parity(p, dtype, variant):
    c = comm(p)
    c.set_option("copy_variant", variant)
    try:
        for m, off in ((1, 0), (7, 1), (4099, 0), (300001, 3)):
            n = p * m
            x = as_dtype(make_inputs("int24", 1, n, "int32", f"sc.{p}.{m}")[0], dtype)
            root = (p - 1) // 2
            src = [Guarded(n, dtype, offset=off, fill=x) if r == root else None for r in range(p)]
            out = [Guarded(m, dtype, offset=(r + off) % 4) for r in range(p)]
            c.scatter([s.t if s else None for s in src], [o.t for o in out], root, n=n, dtype=dtype)
            torch.cuda.synchronize()
            assert c.async_error() == SC.OK
            want = O.scatter(x, p, dtype, root)
            for r in range(p):
                assert out[r].guards_intact()
                np.testing.assert_array_equal(out[r].numpy(), want[r])
            shards = [as_dtype(make_inputs("int24", 1, m, "int32", f"ga.{p}.{m}.{r}")[0], dtype) for r in range(p)]
            gsrc = [Guarded(m, dtype, offset=(r * 3 + off) % 4, fill=shards[r]) for r in range(p)]
            gout = [Guarded(n, dtype, offset=off) if r == root else Guarded(n, dtype) for r in range(p)]
            c.gather([g.t for g in gsrc], [g.t for g in gout], root)
            torch.cuda.synchronize()
            assert c.async_error() == SC.OK
            np.testing.assert_array_equal(gout[root].numpy(), O.gather(shards, dtype, root))
            untouched = Guarded(n, dtype).numpy()
            for r in range(p):
                assert gout[r].guards_intact()
                if r != root:
                    np.testing.assert_array_equal(gout[r].numpy(), untouched)
    finally:
        c.set_option("copy_variant", -1)


def test_scatter_gather_in_place_and_errors():
    p, m = 4, 1000
    n = p * m
    c = comm(p)
    x = make_inputs("int24", 1, n, "int32", "scip")[0]
    root = 2
    buf = to_torch(x, "int32")
    outs = [torch.zeros(m, dtype=torch.int32, device="cuda") for _ in range(p)]
    outs[root] = buf[root * m:(root + 1) * m]           # in place: recv[root] = send[root] + root*m
    c.scatter([None, None, buf, None], outs, root)
    torch.cuda.synchronize()
    for r in range(p):
        np.testing.assert_array_equal(outs[r].cpu().numpy(), x[r * m:(r + 1) * m])
    shards = [make_inputs("int24", 1, m, "int32", f"gaip.{r}")[0] for r in range(p)]
    g = torch.zeros(n, dtype=torch.int32, device="cuda")
    g[root * m:(root + 1) * m] = to_torch(shards[root], "int32")
    sends = [to_torch(s, "int32") for s in shards]
    sends[root] = g[root * m:(root + 1) * m]            # in place: send[root] = recv[root] + root*m
    c.gather(sends, [None, None, g, None], root)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g.cpu().numpy(), np.concatenate(shards))
    with pytest.raises(SC.SimCommError) as e:
        c.scatter([None, None, buf, None], outs, root, algo="ring")
    assert e.value.status == SC.UNSUPPORTED
    with pytest.raises(SC.SimCommError) as e:
        c.gather(sends, [None, None, g, None], 4, n=n)
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:  # Scatter output overlapping the root's input off the in-place form
        c.scatter([None, None, buf, None], [buf[:m], outs[1], outs[2], outs[3]], root)
    assert e.value.status == SC.INVALID_ARG
