"""GPU parity of every collective against the CPU oracle, through the C ABI.

Bars: bit-exact for int32, MIN/MAX and every copy collective; for fp32/bf16 sums the direct path
equals the oracle's rank-order fp32 fold bit for bit and the ring path equals the oracle's ring
emulation bit for bit, and both stay within the stated error bounds of the exact sum.
"""
import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import Guarded, check_sum_tolerance, make_inputs, to_torch

pytestmark = pytest.mark.gpu

PS = [1, 2, 3, 4, 5, 8, 16]
DTYPES = ["int32", "fp32", "bf16"]
_COMMS = {}


def comm(p):
    if p not in _COMMS:
        _COMMS[p] = SC.SimComm(p)
    c = _COMMS[p]
    c.set_option("chunk_bytes", 1 << 20)
    c.set_option("fault_skip_rank", -1)
    c.set_option("timeout_ns", 2_000_000_000)
    c.set_option("copy_variant", -1)
    c.set_option("copy_order", -1)
    return c


def data_kind(dtype, op):
    # integer-valued data keep every fp order exact; "normal" data exercise rounding
    return "int24" if dtype == "int32" else "normal"


def finish(c, bufs):
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    for b in bufs:
        assert b.guards_intact(), "a guard band was overwritten"


def expected_reduction(kind, ins, dtype, op, algo, root=0):
    exactish = dtype == "int32" or op in ("min", "max")
    if algo == "ring":
        if kind == "allreduce":
            return O.ring_allreduce(ins, dtype, op)
        if kind == "reduce_scatter":
            return O.ring_reduce_scatter(ins, dtype, op)
        return O.ring_reduce(ins, dtype, op, root)
    acc = "exact" if exactish else "rankfold"
    if kind == "allreduce":
        return O.allreduce(ins, dtype, op, acc=acc)
    if kind == "reduce_scatter":
        return O.reduce_scatter(ins, dtype, op, acc=acc)
    return O.reduce(ins, dtype, op, root, acc=acc)


# ---- the pages' worked example and figures ----------------------------------------------------------

@pytest.mark.parametrize("algo", ["direct", "ring"])
@pytest.mark.parametrize("dtype", DTYPES)
def test_worked_reduce_example(algo, dtype):
    """[1 2],[3 4],[0 1],[6 7] -> root r0 [10 14] (Reduce) and every rank [10 14] (AllReduce)."""
    c = comm(4)
    vals = [[1, 2], [3, 4], [0, 1], [6, 7]]
    ins = [np.array(v, np.float32) for v in vals]
    if dtype == "int32":
        ins = [x.astype(np.int32) for x in ins]
    elif dtype == "bf16":
        ins = [O.float_to_bf16(x) for x in ins]
    src = [Guarded(2, dtype, fill=x) for x in ins]
    out = [Guarded(2, dtype) for _ in range(4)]
    c.reduce([b.t for b in src], [b.t for b in out], 0, op="sum", algo=algo)
    finish(c, src + out)
    got = out[0].numpy()
    want = np.array([10, 14], np.float32)
    assert list(O.bf16_to_float(got) if dtype == "bf16" else got.astype(np.float32)) == list(want)
    for r in (1, 2, 3):  # the other ranks' outputs are untouched
        assert out[r].guards_intact() and np.array_equal(out[r].numpy(), Guarded(2, dtype).numpy())
    out2 = [Guarded(2, dtype) for _ in range(4)]
    c.allreduce([b.t for b in src], [b.t for b in out2], op="sum", algo=algo)
    finish(c, out2)
    for b in out2:
        g = b.numpy()
        assert list(O.bf16_to_float(g) if dtype == "bf16" else g.astype(np.float32)) == list(want)


# ---- config 1: p = 4, n = 65,536 fp32 integers in [-8, 8] ------------------------------------------

TINY_P, TINY_N = 4, 65536


@pytest.fixture(scope="module")
def tiny():
    return make_inputs("int8", TINY_P, TINY_N, "fp32", "tiny")


@pytest.mark.parametrize("algo", ["direct", "ring"])
@pytest.mark.parametrize("op", ["sum", "min", "max"])
def test_tiny_allreduce(tiny, algo, op):
    c = comm(TINY_P)
    src = [Guarded(TINY_N, "fp32", fill=x) for x in tiny]
    out = [Guarded(TINY_N, "fp32") for _ in tiny]
    c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
    finish(c, src + out)
    want = O.allreduce(tiny, "fp32", op)
    for r in range(TINY_P):
        np.testing.assert_array_equal(out[r].numpy(), want[r])
        np.testing.assert_array_equal(src[r].numpy(), tiny[r])  # inputs untouched


@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_tiny_reduce_broadcast_root2(tiny, algo):
    c = comm(TINY_P)
    src = [Guarded(TINY_N, "fp32", fill=x) for x in tiny]
    out = [Guarded(TINY_N, "fp32") for _ in tiny]
    c.reduce([b.t for b in src], [b.t for b in out], 2, op="sum", algo=algo)
    finish(c, src + out)
    np.testing.assert_array_equal(out[2].numpy(), O.reduce(tiny, "fp32", "sum", 2))
    untouched = Guarded(TINY_N, "fp32").numpy()
    for r in (0, 1, 3):
        np.testing.assert_array_equal(out[r].numpy(), untouched)
    bout = [Guarded(TINY_N, "fp32") for _ in tiny]
    c.broadcast([b.t for b in src], [b.t for b in bout], 2, algo=algo)
    finish(c, bout)
    for r, w in enumerate(O.broadcast(tiny[2], TINY_P, "fp32", 2)):
        np.testing.assert_array_equal(bout[r].numpy(), w)


@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_tiny_reduce_scatter_allgather_alltoall(tiny, algo):
    c = comm(TINY_P)
    m = TINY_N // TINY_P
    src = [Guarded(TINY_N, "fp32", fill=x) for x in tiny]
    rs = [Guarded(m, "fp32") for _ in tiny]
    c.reduce_scatter([b.t for b in src], [b.t for b in rs], op="sum", algo=algo)
    finish(c, src + rs)
    for r, w in enumerate(O.reduce_scatter(tiny, "fp32", "sum")):
        np.testing.assert_array_equal(rs[r].numpy(), w)
    shards = [x[:m].copy() for x in tiny]
    sh = [Guarded(m, "fp32", fill=x) for x in shards]
    ag = [Guarded(TINY_N, "fp32") for _ in tiny]
    c.allgather([b.t for b in sh], [b.t for b in ag], algo=algo)
    finish(c, sh + ag)
    for r, w in enumerate(O.allgather(shards, "fp32")):
        np.testing.assert_array_equal(ag[r].numpy(), w)
    a2a = [Guarded(TINY_N, "fp32") for _ in tiny]
    c.alltoall([b.t for b in src], [b.t for b in a2a], algo=algo)
    finish(c, a2a)
    for r, w in enumerate(O.alltoall(tiny, "fp32")):
        np.testing.assert_array_equal(a2a[r].numpy(), w)


# ---- reductions over p, dtype, op, size, alignment -----------------------------------------------

def sizes(p, divisible):
    base = [1, 7, 999, 4099, 70001]
    if divisible:
        return [p * k for k in (1, 3, 64, 1001, 16411)]
    return base


@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("op", ["sum", "min", "max", "avg"])
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_allreduce_parity(p, dtype, op, algo):
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    if algo == "ring":
        c.set_option("chunk_bytes", 1024)  # many chunks per segment: exercises the pipeline
    for n in sizes(p, False):
        ins = make_inputs(data_kind(dtype, op), p, n, dtype, f"ar.{p}.{n}", sigma=1e-3)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(n, dtype) for _ in ins]
        c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
        finish(c, src + out)
        want = expected_reduction("allreduce", ins, dtype, op, algo)
        for r in range(p):
            got = out[r].numpy()
            np.testing.assert_array_equal(got, want[r], err_msg=f"n={n} rank={r}")
        if dtype != "int32" and op in ("sum", "avg"):
            check_sum_tolerance(out[0].numpy(), ins, dtype, op, p)


@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("op", ["sum", "max", "avg"])
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_reduce_scatter_and_reduce_parity(p, dtype, op, algo):
    if dtype == "int32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    c = comm(p)
    if algo == "ring":
        c.set_option("chunk_bytes", 512)
    for n in sizes(p, True):
        m = n // p
        ins = make_inputs(data_kind(dtype, op), p, n, dtype, f"rs.{p}.{n}", sigma=1e-2)
        src = [Guarded(n, dtype, fill=x) for x in ins]
        out = [Guarded(m, dtype) for _ in ins]
        c.reduce_scatter([b.t for b in src], [b.t for b in out], op=op, algo=algo)
        finish(c, src + out)
        want = expected_reduction("reduce_scatter", ins, dtype, op, algo)
        for r in range(p):
            np.testing.assert_array_equal(out[r].numpy(), want[r], err_msg=f"n={n} rank={r}")
        root = p - 1
        rout = [Guarded(n, dtype) for _ in ins]
        c.reduce([b.t for b in src], [b.t for b in rout], root, op=op, algo=algo)
        finish(c, rout)
        np.testing.assert_array_equal(rout[root].numpy(), expected_reduction("reduce", ins, dtype, op, algo, root))
        if dtype != "int32" and op != "max":
            check_sum_tolerance(rout[root].numpy(), ins, dtype, op, p)


@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_copy_collectives_parity(p, dtype, algo):
    c = comm(p)
    if algo == "ring":
        c.set_option("chunk_bytes", 768)
    for n in sizes(p, True) + [p * 300000]:
        m = n // p
        ins = make_inputs("int24", p, n, "int32", f"cp.{p}.{n}")
        if dtype != "int32":
            ins = [x.view(np.float32).copy() if dtype == "fp32" else x.astype(np.uint16) for x in ins]
        src = [Guarded(n, dtype, fill=x) for x in ins]
        # Broadcast from the last rank
        out = [Guarded(n, dtype) for _ in ins]
        c.broadcast([b.t for b in src], [b.t for b in out], p - 1, algo=algo)
        finish(c, src + out)
        for r in range(p):
            np.testing.assert_array_equal(out[r].numpy(), ins[p - 1])
        # AllGather of the first m elements
        shards = [x[:m].copy() for x in ins]
        sh = [Guarded(m, dtype, fill=x) for x in shards]
        ag = [Guarded(n, dtype) for _ in ins]
        c.allgather([b.t for b in sh], [b.t for b in ag], algo=algo)
        finish(c, sh + ag)
        for r, w in enumerate(O.allgather(shards, dtype)):
            np.testing.assert_array_equal(ag[r].numpy(), w)
        # All-to-All, and back
        a2a = [Guarded(n, dtype) for _ in ins]
        c.alltoall([b.t for b in src], [b.t for b in a2a], algo=algo)
        finish(c, a2a)
        want = O.alltoall(ins, dtype)
        for r in range(p):
            np.testing.assert_array_equal(a2a[r].numpy(), want[r])
        back = [Guarded(n, dtype) for _ in ins]
        c.alltoall([b.t for b in a2a], [b.t for b in back], algo=algo)
        finish(c, back)
        for r in range(p):
            np.testing.assert_array_equal(back[r].numpy(), ins[r])


@pytest.mark.parametrize("p", [2, 3, 8])
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_unaligned_buffers(p, dtype, algo):
    """Buffers one element off a 16-byte boundary take the element-wise paths: same results."""
    c = comm(p)
    n = p * 5003
    m = n // p
    ins = make_inputs("normal" if dtype != "int32" else "int24", p, n, dtype, f"ua.{p}", sigma=1e-2)
    src = [Guarded(n, dtype, offset=1, fill=x) for x in ins]
    out = [Guarded(n, dtype, offset=1) for _ in ins]
    op = "max" if dtype == "int32" else "sum"
    c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
    finish(c, src + out)
    want = expected_reduction("allreduce", ins, dtype, op, algo)
    for r in range(p):
        np.testing.assert_array_equal(out[r].numpy(), want[r])
    rs = [Guarded(m, dtype, offset=3) for _ in ins]
    c.reduce_scatter([b.t for b in src], [b.t for b in rs], op=op, algo=algo)
    finish(c, rs)
    want = expected_reduction("reduce_scatter", ins, dtype, op, algo)
    for r in range(p):
        np.testing.assert_array_equal(rs[r].numpy(), want[r])
    a2a = [Guarded(n, dtype, offset=r % 3) for r in range(p)]
    c.alltoall([b.t for b in src], [b.t for b in a2a], algo=algo)
    finish(c, a2a)
    want = O.alltoall(ins, dtype)
    for r in range(p):
        np.testing.assert_array_equal(a2a[r].numpy(), want[r])
    shards = [x[:m].copy() for x in ins]
    sh = [Guarded(m, dtype, offset=(r + 1) % 4, fill=shards[r]) for r in range(p)]
    ag = [Guarded(n, dtype, offset=2) for _ in ins]
    c.allgather([b.t for b in sh], [b.t for b in ag], algo=algo)
    finish(c, sh + ag)
    for r, w in enumerate(O.allgather(shards, dtype)):
        np.testing.assert_array_equal(ag[r].numpy(), w)


# ---- in place ----------------------------------------------------------------------------------

@pytest.mark.parametrize("algo", ["direct", "ring"])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_in_place_forms(algo, dtype):
    p, n = 4, 4 * 20000
    m = n // p
    c = comm(p)
    c.set_option("chunk_bytes", 4096)
    ins = make_inputs("normal", p, n, dtype, "inplace", sigma=1e-2)
    # AllReduce: send == recv
    bufs = [Guarded(n, dtype, fill=x) for x in ins]
    c.allreduce([b.t for b in bufs], [b.t for b in bufs], op="sum", algo=algo)
    finish(c, bufs)
    want = expected_reduction("allreduce", ins, dtype, "sum", algo)
    for r in range(p):
        np.testing.assert_array_equal(bufs[r].numpy(), want[r])
    # ReduceScatter: recv[r] = send[r] + r*m
    bufs = [Guarded(n, dtype, fill=x) for x in ins]
    c.reduce_scatter([b.t for b in bufs], [bufs[r].t[r * m:(r + 1) * m] for r in range(p)], op="sum", algo=algo)
    finish(c, bufs)
    want = expected_reduction("reduce_scatter", ins, dtype, "sum", algo)
    for r in range(p):
        np.testing.assert_array_equal(bufs[r].numpy()[r * m:(r + 1) * m], want[r])
    # AllGather: send[r] = recv[r] + r*m
    shards = [x[:m].copy() for x in ins]
    bufs = [Guarded(n, dtype) for _ in ins]
    for r in range(p):
        bufs[r].t[r * m:(r + 1) * m].copy_(to_torch(shards[r], dtype))
    c.allgather([bufs[r].t[r * m:(r + 1) * m] for r in range(p)], [b.t for b in bufs], algo=algo)
    finish(c, bufs)
    for r, w in enumerate(O.allgather(shards, dtype)):
        np.testing.assert_array_equal(bufs[r].numpy(), w)
    # Reduce and Broadcast: the root's send == recv
    bufs = [Guarded(n, dtype, fill=x) for x in ins]
    c.reduce([b.t for b in bufs], [None, bufs[1].t, None, None], 1, op="sum", algo=algo)
    finish(c, bufs)
    np.testing.assert_array_equal(bufs[1].numpy(), expected_reduction("reduce", ins, dtype, "sum", algo, 1))
    np.testing.assert_array_equal(bufs[0].numpy(), ins[0])
    bufs = [Guarded(n, dtype, fill=x) for x in ins]
    c.broadcast([None, None, bufs[2].t, None], [b.t for b in bufs], 2, algo=algo)
    finish(c, bufs)
    for r in range(p):
        np.testing.assert_array_equal(bufs[r].numpy(), ins[2])


# ---- All-to-Allv ---------------------------------------------------------------------------------

@pytest.mark.parametrize("p", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_alltoallv_parity_and_inverse(p, dtype, algo):
    c = comm(p)
    if algo == "ring":
        c.set_option("chunk_bytes", 1024)
    rng = np.random.default_rng(1000 * p + len(dtype))
    for scale in (1, 37, 4096):
        counts = rng.integers(0, 6, size=(p, p)) * scale + rng.integers(0, 3, size=(p, p))
        counts[rng.random((p, p)) < 0.25] = 0
        rows = counts.sum(axis=1)
        ins = [make_inputs("int24", 1, int(rows[i]), "int32", f"a2av.{p}.{i}.{scale}")[0] for i in range(p)]
        if dtype == "fp32":
            ins = [x.view(np.float32).copy() for x in ins]
        elif dtype == "bf16":
            ins = [x.astype(np.uint16) for x in ins]
        cap = int(counts.sum(axis=0).max()) + 5
        src = [Guarded(int(rows[i]), dtype, fill=ins[i]) for i in range(p)]
        dst = [Guarded(cap, dtype) for _ in range(p)]
        cnt = torch.tensor(counts, dtype=torch.int64, device="cuda")
        rc = torch.full((p,), -1, dtype=torch.int64, device="cuda")
        c.alltoallv([b.t for b in src], [b.t for b in dst], cnt, algo=algo, recv_counts=rc)
        finish(c, src + dst)
        want, want_rc = O.alltoallv(ins, counts, dtype)
        np.testing.assert_array_equal(rc.cpu().numpy(), want_rc)
        for j in range(p):
            got = dst[j].numpy()
            np.testing.assert_array_equal(got[:want[j].size], want[j])
            # beyond the received elements the buffer is untouched
            np.testing.assert_array_equal(got[want[j].size:], Guarded(cap, dtype).numpy()[want[j].size:])
        # combine: the transposed counts bring every element home
        back = [Guarded(int(rows[i]), dtype) for i in range(p)]
        cntT = torch.tensor(np.ascontiguousarray(counts.T), dtype=torch.int64, device="cuda")
        c.alltoallv([dst[j].t for j in range(p)], [b.t for b in back], cntT, algo=algo)
        finish(c, back)
        for i in range(p):
            np.testing.assert_array_equal(back[i].numpy(), ins[i])


# ---- determinism, errors, failure handling ---------------------------------------------------------

@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_repeated_runs_are_bit_identical(algo):
    p, n = 8, 8 * 50021
    c = comm(p)
    c.set_option("chunk_bytes", 8192)
    ins = make_inputs("normal", p, n, "fp32", "det", sigma=1.0)
    src = [Guarded(n, "fp32", fill=x) for x in ins]
    outs = []
    for _ in range(10):
        out = [Guarded(n, "fp32") for _ in range(p)]
        c.allreduce([b.t for b in src], [b.t for b in out], op="sum", algo=algo)
        finish(c, out)
        outs.append(out[3].numpy())
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])


def test_synchronous_argument_errors():
    p = 4
    c = comm(p)
    t = [torch.zeros(64, device="cuda") for _ in range(p)]
    u = [torch.zeros(64, device="cuda") for _ in range(p)]
    with pytest.raises(SC.SimCommError) as e:
        c.reduce(t, u, 4)
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:
        c.broadcast(t, u, -1)
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:
        c.reduce_scatter(t, [x[:16] for x in u], n=63)
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:
        c.allreduce([x.int() for x in t], [x.int() for x in u], op="avg")
    assert e.value.status == SC.UNSUPPORTED
    with pytest.raises(SC.SimCommError) as e:  # two ranks write the same output
        c.allreduce(t, [u[0], u[0], u[2], u[3]])
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:  # an output overlaps another rank's input
        c.allreduce(t, [t[1], u[1], u[2], u[3]])
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:  # All-to-All is never in place
        c.alltoall(t, t)
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:  # ReduceScatter in place at the wrong offset
        c.reduce_scatter(t, [t[r][:16] for r in range(p)])
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:
        c.allreduce([None] * p, u, n=64)
    assert e.value.status == SC.INVALID_ARG
    with pytest.raises(SC.SimCommError) as e:
        c.set_option("chunk_bytes", 100)
    assert e.value.status == SC.INVALID_ARG
    # zero-sized calls are no-ops
    c.allreduce(t, u, n=0)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK


@pytest.mark.parametrize("p", [1, 4, 6])
def test_zero_size_calls_are_no_ops(p):
    """n = 0 (and an All-to-Allv of all-zero counts) is accepted by every collective and schedule and
    touches no input or output; the All-to-Allv reports zero received elements."""
    c = comm(p)
    t = [torch.full((64,), 3.0, device="cuda") for _ in range(p)]
    u = [torch.full((64,), 7.0, device="cuda") for _ in range(p)]
    pow2 = p & (p - 1) == 0
    for algo in ("direct", "ring", "tree", "dbtree", "ll", "tree_ll", "dbtree_ll") + (("rd", "hd", "rd_ll") if pow2 else ()):
        for op in ("sum", "max"):
            c.allreduce(t, u, op=op, algo=algo, n=0)
    for algo in ("direct", "ring"):
        c.reduce(t, u, p - 1, algo=algo, n=0)
        c.broadcast(t, u, 0, algo=algo, n=0)
        c.reduce_scatter(t, u, algo=algo, n=0)
        c.allgather(t, u, algo=algo, n=0)
        c.alltoall(t, u, algo=algo, n=0)
        rc = torch.full((p,), -1, dtype=torch.int64, device="cuda")
        c.alltoallv(t, u, torch.zeros((p, p), dtype=torch.int64, device="cuda"), algo=algo, recv_counts=rc)
        torch.cuda.synchronize()
        assert torch.equal(rc, torch.zeros_like(rc)), algo
    c.reduce_scatter(t, u, algo="ll", n=0)
    c.allgather(t, u, algo="ll", n=0)
    c.scatter(t, u, 0, n=0)
    c.gather(t, u, 0, n=0)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    assert all(torch.equal(x, torch.full_like(x, 7.0)) for x in u)
    assert all(torch.equal(x, torch.full_like(x, 3.0)) for x in t)


@pytest.mark.parametrize("hint", [-1, 0, 1, 2])
def test_l2_policies_change_no_result(hint):
    """Every L2 policy of option l2_hint (per path, none, evict-first loads and stores on the direct
    paths, evict-first stores on the bulk copies) gives the oracle's results on the fused reduction's
    32-byte path and the copy paths."""
    p, n = 8, 8 * 65544
    c = comm(p)
    c.set_option("l2_hint", hint)
    try:
        ins = make_inputs("int24", p, n, "int32", f"l2.{hint}")
        src = [Guarded(n, "int32", fill=x) for x in ins]
        out = [Guarded(n, "int32") for _ in ins]
        c.allreduce([b.t for b in src], [b.t for b in out], op="sum")
        finish(c, src + out)
        want = O.allreduce(ins, "int32", "sum")
        for r in range(p):
            np.testing.assert_array_equal(out[r].numpy(), want[r])
        c.reduce_scatter([b.t for b in src], [b.t[: n // p] for b in out], op="max")
        finish(c, out)
        want = O.reduce_scatter(ins, "int32", "max")
        for r in range(p):
            np.testing.assert_array_equal(out[r].numpy()[: n // p], want[r])
        c.broadcast([b.t for b in src], [b.t for b in out], 3)
        finish(c, out)
        for r in range(p):
            np.testing.assert_array_equal(out[r].numpy(), ins[3])
        c.alltoall([b.t for b in src], [b.t for b in out])
        finish(c, out)
        for r, w in enumerate(O.alltoall(ins, "int32")):
            np.testing.assert_array_equal(out[r].numpy(), w)
    finally:
        c.set_option("l2_hint", -1)


def test_alltoallv_overflow_is_reported_and_nothing_is_copied():
    p = 3
    c = comm(p)
    counts = np.array([[1, 2, 3], [4, 5, 6], [7, 8, 900]], np.int64)
    src = [Guarded(int(counts[i].sum()), "fp32", fill=np.arange(counts[i].sum(), dtype=np.float32))
           for i in range(p)]
    dst = [Guarded(100, "fp32") for _ in range(p)]
    c.alltoallv([b.t for b in src], [b.t for b in dst], torch.tensor(counts, device="cuda"))
    torch.cuda.synchronize()
    assert c.async_error() == SC.OVERFLOW
    untouched = Guarded(100, "fp32").numpy()
    for b in dst:
        np.testing.assert_array_equal(b.numpy(), untouched)
    with pytest.raises(SC.SimCommError) as e:  # sticky until reset
        c.allreduce([b.t[:4] for b in dst], [b.t[4:8] for b in dst])
    assert e.value.status == SC.OVERFLOW
    c.reset()
    assert c.async_error() == SC.OK
    ok = torch.tensor(np.minimum(counts, 9), device="cuda")
    c.alltoallv([b.t for b in src], [b.t for b in dst], ok)
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK


@pytest.mark.parametrize("kind", ["allreduce", "reduce", "broadcast", "allgather"])
def test_ring_timeout_when_a_rank_never_signals(kind):
    """Host-side fault injection: rank 1's steps are never signalled, so its successor's bounded
    wait gives up and the call reports COLL_ERR_TIMEOUT; reset makes the communicator usable."""
    p, n = 4, 4 * 4096
    c = comm(p)
    c.set_option("chunk_bytes", 4096)
    c.set_option("timeout_ns", 200_000_000)
    c.set_option("fault_skip_rank", 1)
    t = [torch.ones(n, device="cuda") for _ in range(p)]
    u = [torch.zeros(n, device="cuda") for _ in range(p)]
    if kind == "allreduce":
        c.allreduce(t, u, algo="ring")
    elif kind == "reduce":
        c.reduce(t, u, 3, algo="ring")
    elif kind == "broadcast":
        c.broadcast(t, u, 0, algo="ring")
    else:
        c.allgather([x[:n // p] for x in t], u, algo="ring")
    torch.cuda.synchronize()
    assert c.async_error() == SC.TIMEOUT
    c.set_option("fault_skip_rank", -1)
    c.reset()
    c.allreduce(t, u, algo="ring")
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    assert torch.equal(u[2], torch.full_like(u[2], float(p)))


def test_abort_stops_a_waiting_ring_step():
    import time
    p, n = 4, 4 * 4096
    c = comm(p)
    c.set_option("chunk_bytes", 4096)
    c.set_option("timeout_ns", 5_000_000_000)
    c.set_option("fault_skip_rank", 2)
    t = [torch.ones(n, device="cuda") for _ in range(p)]
    u = [torch.zeros(n, device="cuda") for _ in range(p)]
    t0 = time.time()
    c.allreduce(t, u, algo="ring")
    time.sleep(0.05)
    c.abort()
    torch.cuda.synchronize()
    assert time.time() - t0 < 4.0
    assert c.async_error() == SC.ABORTED
    with pytest.raises(SC.SimCommError) as e:
        c.allreduce(t, u, algo="ring")
    assert e.value.status == SC.ABORTED
    c.set_option("fault_skip_rank", -1)
    c.reset()
    c.allreduce(t, u, algo="ring")
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK


def test_launch_count_counts_kernels():
    c = comm(2)
    before = c.launch_count()
    t = [torch.ones(256, device="cuda") for _ in range(2)]
    u = [torch.zeros(256, device="cuda") for _ in range(2)]
    c.allreduce(t, u)
    c.allreduce(t, u, algo="ring")
    c.allgather([x[:128] for x in t], u)
    torch.cuda.synchronize()
    assert c.launch_count() - before == 3


@pytest.mark.parametrize("order", [-1, 0, 1])
@pytest.mark.parametrize("variant", list(range(-1, 19)))
@pytest.mark.parametrize("p", [3, 8])
def test_copy_engine_variants(variant, p, order):
    """Every copy path (the per-collective default, each bulk-copy pipeline shape, the load/store
    path and the lean copies of Broadcast, AllGather and All-to-All, with and without lagged stage
    reuse) in both tile orders gives the oracle's results. The lean copies need 16-byte aligned
    buffers and whole 16-byte (one-pass: 32-byte) blocks, as in the 65,544-element case with its
    short last tile; the others fall back."""
    c = comm(p)
    c.set_option("copy_variant", variant)
    c.set_option("copy_order", order)
    try:
        for n, off in ((p * 7, 0), (p * 40961, 1), (p * 300007, 0), (p * 65544, 0)):
            m = n // p
            ins = make_inputs("int24", p, n, "int32", f"cv.{p}.{n}")
            src = [Guarded(n, "int32", offset=off, fill=x) for x in ins]
            out = [Guarded(n, "int32") for _ in ins]
            c.broadcast([b.t for b in src], [b.t for b in out], 1, algo="direct")
            finish(c, src + out)
            for r in range(p):
                np.testing.assert_array_equal(out[r].numpy(), ins[1])
            shards = [x[:m].copy() for x in ins]
            sh = [Guarded(m, "int32", offset=off, fill=x) for x in shards]
            ag = [Guarded(n, "int32", offset=off) for _ in ins]
            c.allgather([b.t for b in sh], [b.t for b in ag], algo="direct")
            finish(c, sh + ag)
            for r, w in enumerate(O.allgather(shards, "int32")):
                np.testing.assert_array_equal(ag[r].numpy(), w)
            a2a = [Guarded(n, "int32") for _ in ins]
            c.alltoall([b.t for b in src], [b.t for b in a2a], algo="direct")
            finish(c, a2a)
            for r, w in enumerate(O.alltoall(ins, "int32")):
                np.testing.assert_array_equal(a2a[r].numpy(), w)
            counts = np.random.default_rng(n).integers(0, m // p + 3, size=(p, p))
            rows = counts.sum(axis=1)
            vsrc = [Guarded(int(rows[i]), "int32", fill=ins[i][:rows[i]]) for i in range(p)]
            cap = int(counts.sum(axis=0).max())
            vdst = [Guarded(cap, "int32") for _ in range(p)]
            c.alltoallv([b.t for b in vsrc], [b.t for b in vdst], torch.tensor(counts, device="cuda"), algo="direct")
            finish(c, vsrc + vdst)
            want, _ = O.alltoallv([ins[i][:rows[i]] for i in range(p)], counts, "int32")
            for j in range(p):
                np.testing.assert_array_equal(vdst[j].numpy()[:want[j].size], want[j])
    finally:
        c.set_option("copy_variant", -1)
        c.set_option("copy_order", -1)


@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("variant", [-1, 0, 4, 8])
def test_alltoallv_skewed_blocks_every_order(variant, order):
    """Hot-destination counts (one column far larger than the rest, some blocks empty): the
    interleaved order's level table gives every task exactly once."""
    p, m = 8, 300007
    c = comm(p)
    c.set_option("copy_variant", variant)
    c.set_option("copy_order", order)
    try:
        ins = make_inputs("int24", p, m, "int32", f"skew.{p}")
        counts = np.zeros((p, p), dtype=np.int64)
        for i in range(p):
            counts[i, 0] = m // 2 + 977 * i
            for j in range(1, p):
                counts[i, j] = 0 if (i + j) % 4 == 0 else 1031 * ((i * 3 + j) % 5) + 13
        rows = counts.sum(axis=1)
        assert rows.max() <= m
        vsrc = [Guarded(int(rows[i]), "int32", fill=ins[i][:rows[i]]) for i in range(p)]
        cap = int(counts.sum(axis=0).max())
        vdst = [Guarded(cap, "int32") for _ in range(p)]
        rc = torch.zeros(p, dtype=torch.int64, device="cuda")
        c.alltoallv([b.t for b in vsrc], [b.t for b in vdst], torch.tensor(counts, device="cuda"), algo="direct",
                    recv_counts=rc)
        finish(c, vsrc + vdst)
        want, _ = O.alltoallv([ins[i][:rows[i]] for i in range(p)], counts, "int32")
        for j in range(p):
            np.testing.assert_array_equal(vdst[j].numpy()[:want[j].size], want[j])
        assert rc.cpu().tolist() == counts.sum(axis=0).tolist()
    finally:
        c.set_option("copy_variant", -1)
        c.set_option("copy_order", -1)


def test_alltoallv_interleaved_beyond_the_level_table():
    """A block of more tiles than the level table holds (over 8,192 tiles of 16 KiB): the interleaved
    order falls back to skipping empty slots and still gives the oracle's result."""
    p = 2
    c = comm(p)
    c.set_option("copy_variant", 4)  # 16 KiB tiles
    c.set_option("copy_order", 1)
    try:
        big = 8300 * 4096 + 5  # int32 elements: 8,301 tiles
        counts = np.array([[3, big], [7, 11]], dtype=np.int64)
        rows = counts.sum(axis=1)
        ins = [make_inputs("int24", 1, int(rows[i]), "int32", f"lvl.big.{i}")[0] for i in range(p)]
        vsrc = [torch.from_numpy(x).cuda() for x in ins]
        cols = counts.sum(axis=0)
        vdst = [torch.zeros(int(cols[j]), dtype=torch.int32, device="cuda") for j in range(p)]
        c.alltoallv(vsrc, vdst, torch.tensor(counts, device="cuda"), algo="direct")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        want, _ = O.alltoallv(ins, counts, "int32")
        for j in range(p):
            np.testing.assert_array_equal(vdst[j].cpu().numpy(), want[j])
    finally:
        c.set_option("copy_variant", -1)
        c.set_option("copy_order", -1)
