"""Pins of the CPU oracle against what the pages and the mathematics fix.

The oracle must not be trusted on its own say-so: every function is checked here against the
pages' worked example and figure layouts (tests/golden/), against closed forms and identities
stated on the pages, and against library routines (numpy concatenate/transpose/split/sum,
math.fsum, exact rational rounding) on brute-force tiny inputs.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PS = [1, 2, 3, 4, 5, 7, 8]


# ----------------------------------------------------------------------------------------------
# helpers (library routines only)

def rng_ints(seed, p, n, lo=-8, hi=8):
    r = np.random.default_rng(seed)
    return [r.integers(lo, hi + 1, size=n).astype(np.int32) for _ in range(p)]


def rng_f32(seed, p, n, scale=1.0):
    r = np.random.default_rng(seed)
    return [(r.standard_normal(n) * scale).astype(np.float32) for _ in range(p)]


def bf16_bits_from_f32(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def bf16_to_f32(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def exact_round_bf16(fr: Fraction) -> float:
    """Round an exact rational to the nearest bf16 (8 significant bits), ties to even."""
    if fr == 0:
        return 0.0
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** max(e - 7, -133)
    t = a / q
    fl = t.numerator // t.denominator
    rem = t - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * float(fl * q)


def fsum_f32(vals):
    return np.float32(math.fsum(float(v) for v in vals))


def wrap_i32(x):
    return np.asarray(x, dtype=np.int64).astype(np.int32)


# ----------------------------------------------------------------------------------------------
# golden fixtures

def parse_worked():
    d = {"in": {}}
    for line in open(os.path.join(GOLDEN, "worked_reduce.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        key, _, rest = line.partition(":") if ":" in line else (line.split()[0], None, " ".join(line.split()[1:]))
        if key.startswith("in "):
            d["in"][int(key.split()[1])] = [int(v) for v in rest.split()]
        elif key in ("p", "root"):
            d[key] = int(rest)
        else:
            d[key] = [int(v) for v in rest.split()]
    return d


@pytest.mark.parametrize("dtype", ["fp32", "int32", "bf16"])
@pytest.mark.parametrize("acc", ["exact", "rankfold"])
def test_worked_reduce_example(dtype, acc):
    g = parse_worked()
    p, root = g["p"], g["root"]
    if dtype == "bf16":
        ins = [bf16_bits_from_f32(np.array(g["in"][r], np.float32)) for r in range(p)]
        conv = bf16_to_f32
    else:
        ins = [np.array(g["in"][r], dtype=O.NP_DTYPES[dtype]) for r in range(p)]
        conv = np.asarray
    red = O.reduce(ins, dtype, "sum", root, acc=acc if dtype != "int32" else "exact")
    assert list(conv(red)) == g["reduce_root"]
    for out in O.allreduce(ins, dtype, "sum", acc=acc if dtype != "int32" else "exact"):
        assert list(conv(out)) == g["allreduce"]
    if dtype != "int32" or acc == "exact":
        assert list(conv(O.ring_reduce(ins, dtype, "sum", root))) == g["reduce_root"]
        for out in O.ring_allreduce(ins, dtype, "sum"):
            assert list(conv(out)) == g["allreduce"]


def test_reduce_leaves_nonroot_untouched_and_only_root_written():
    g = parse_worked()
    ins = [np.array(g["in"][r], np.float32) for r in range(g["p"])]
    sentinel = np.full(2, -12345.0, np.float32)
    before = sentinel.copy()
    # the oracle writes exactly one buffer: the one it is given for the root
    out = O.reduce(ins, "fp32", "sum", g["root"], out=sentinel)
    assert out is sentinel and list(out) == g["reduce_root"]
    assert not np.array_equal(before, out)


def parse_figures():
    figs, cur = [], None
    for raw in open(os.path.join(GOLDEN, "layout_figures.txt")):
        line = raw.split("#")[0].strip()
        if not line:
            continue
        if line.startswith("figure"):
            cur = {"name": line.split()[1], "in": {}, "out": {}, "root": None}
        elif line == "end":
            figs.append(cur)
        elif line.startswith("in ") or line.startswith("out "):
            head, rest = line.split(":", 1)
            kind, r = head.split()
            cur[kind][int(r)] = rest.split()
        else:
            k, v = line.split()
            cur[k] = int(v)
    return figs


def symbol_value(sym, table):
    if sym not in table:
        table[sym] = 1 + 37 * len(table) + (len(table) ** 3) % 1009
    return table[sym]


@pytest.mark.parametrize("fig", parse_figures(), ids=lambda f: f["name"])
@pytest.mark.parametrize("ring", [False, True])
def test_layout_figures(fig, ring):
    p = fig["p"]
    table = {}
    ins = []
    for r in range(p):
        vals = [(-99999 - r) if s == "." else symbol_value(s, table) for s in fig["in"][r]]
        ins.append(np.array(vals, np.int32))
    name = fig["name"]
    if name == "broadcast":
        root = fig["root"]
        outs = (O.ring_broadcast if ring else O.broadcast)(ins[root], p, "int32", root)
    elif name == "allgather":
        outs = (O.ring_allgather if ring else O.allgather)(ins, "int32")
    elif name == "reduce_scatter":
        outs = O.ring_reduce_scatter(ins, "int32", "sum") if ring else O.reduce_scatter(ins, "int32", "sum")
    elif name == "alltoall":
        outs = (O.ring_alltoall if ring else O.alltoall)(ins, "int32")
    else:
        raise AssertionError(name)
    for r in range(p):
        want = [sum(table[s] for s in tok.split("+")) for tok in fig["out"][r]]
        assert list(outs[r]) == want, (name, r)


def test_ring_fold_order_golden():
    vals = {}
    for raw in open(os.path.join(GOLDEN, "ring_fold_order.txt")):
        line = raw.split("#")[0].strip()
        if not line:
            continue
        if ":" in line:
            k, v = line.split(":")
            vals[k.strip()] = [float(x) for x in v.split()]
        else:
            k, v = line.split()
            vals[k] = int(v)
    p = vals["p"]
    ins = [np.array(vals[f"in {r}"], np.float32) for r in range(p)]
    for out in O.ring_allreduce(ins, "fp32", "sum"):
        assert list(out) == vals["ring_allreduce"]
    for out in O.allreduce(ins, "fp32", "sum", acc="rankfold"):
        assert list(out) == vals["rank_order_allreduce"]
    # ReduceScatter alone: rank r owns the complete chunk r after p-1 steps
    for r, out in enumerate(O.ring_reduce_scatter(ins, "fp32", "sum")):
        assert list(out) == [vals["ring_allreduce"][r]]


# ----------------------------------------------------------------------------------------------
# brute force against library routines

@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("op", ["sum", "min", "max"])
def test_int32_reductions_bruteforce(p, op):
    for n in (0, 1, p, 3 * p, 1000 * p):
        ins = rng_ints(100 * p + n, p, n, lo=-2**24, hi=2**24)
        stack = np.stack(ins) if n else np.zeros((p, 0), np.int32)
        want = {"sum": lambda: wrap_i32(stack.astype(np.int64).sum(axis=0)),
                "min": lambda: stack.min(axis=0), "max": lambda: stack.max(axis=0)}[op]()
        for out in O.allreduce(ins, "int32", op):
            np.testing.assert_array_equal(out, want)
        for root in {0, p - 1}:
            np.testing.assert_array_equal(O.reduce(ins, "int32", op, root), want)
        if n % p == 0:
            m = n // p
            for r, out in enumerate(O.reduce_scatter(ins, "int32", op)):
                np.testing.assert_array_equal(out, want[r * m:(r + 1) * m])


def test_int32_sum_wraps_twos_complement():
    ins = [np.array([2**31 - 1, -2**31], np.int32), np.array([1, -1], np.int32)]
    out = O.allreduce(ins, "int32", "sum")[0]
    assert list(out) == [-2**31, 2**31 - 1]


@pytest.mark.parametrize("p", PS)
def test_fp32_rankfold_is_sequential_fp32_addition(p):
    n = 997
    ins = rng_f32(7 * p, p, n)
    acc = ins[0].copy()
    for x in ins[1:]:
        acc = (acc + x).astype(np.float32)
    for out in O.allreduce(ins, "fp32", "sum", acc="rankfold"):
        np.testing.assert_array_equal(out, acc)
    scale = np.float32(1.0) / np.float32(p)
    for out in O.allreduce(ins, "fp32", "avg", acc="rankfold"):
        np.testing.assert_array_equal(out, (acc * scale).astype(np.float32))


@pytest.mark.parametrize("p", PS)
def test_fp32_exact_is_correctly_rounded_sum(p):
    n = 301
    ins = rng_f32(11 * p, p, n)
    want = np.array([fsum_f32([x[i] for x in ins]) for i in range(n)], np.float32)
    for out in O.allreduce(ins, "fp32", "sum", acc="exact"):
        np.testing.assert_array_equal(out, want)
    want_avg = np.array([np.float32(math.fsum(float(x[i]) for x in ins) / p) for i in range(n)], np.float32)
    np.testing.assert_array_equal(O.allreduce(ins, "fp32", "avg", acc="exact")[0], want_avg)


@pytest.mark.parametrize("p", [2, 3, 8])
def test_bf16_exact_and_rankfold(p):
    n = 257
    ins32 = rng_f32(13 * p, p, n, scale=1e-2)
    ins = [bf16_bits_from_f32(x) for x in ins32]
    vals = [bf16_to_f32(h) for h in ins]
    exact = O.allreduce(ins, "bf16", "sum", acc="exact")[0]
    for i in range(n):
        fr = sum((Fraction(float(v[i])) for v in vals), Fraction(0))
        assert bf16_to_f32(exact[i:i + 1])[0] == np.float32(exact_round_bf16(fr))
    acc = vals[0].copy()
    for v in vals[1:]:
        acc = (acc + v).astype(np.float32)
    np.testing.assert_array_equal(O.allreduce(ins, "bf16", "sum", acc="rankfold")[0], bf16_bits_from_f32(acc))


@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_avg_is_exact_scaling_for_power_of_two_p(p):
    ins = rng_f32(17 * p, p, 513)
    s = O.allreduce(ins, "fp32", "sum", acc="rankfold")[0]
    a = O.allreduce(ins, "fp32", "avg", acc="rankfold")[0]
    np.testing.assert_array_equal(a, np.ldexp(s, -int(math.log2(p))).astype(np.float32))


def test_minmax_ties_keep_earlier_rank():
    pz, nz = np.float32(0.0), np.float32(-0.0)
    ins = [np.array([nz, pz], np.float32), np.array([pz, nz], np.float32)]
    mn = O.allreduce(ins, "fp32", "min")[0]
    mx = O.allreduce(ins, "fp32", "max")[0]
    assert list(np.signbit(mn)) == [True, False] and list(np.signbit(mx)) == [True, False]


@pytest.mark.parametrize("p", PS)
def test_copy_collectives_bruteforce(p):
    for m in (0, 1, 5, 64):
        n = p * m
        ins = rng_ints(3 * p + m, p, n, lo=-1000, hi=1000)
        # AllGather: concatenation in rank order
        shards = [x[:m].copy() for x in ins]
        for out in O.allgather(shards, "int32"):
            np.testing.assert_array_equal(out, np.concatenate(shards) if m else np.zeros(0, np.int32))
        # All-to-All: transpose of the [src][dst] block matrix
        blocks = np.stack(ins).reshape(p, p, m)
        want = blocks.transpose(1, 0, 2).reshape(p, n)
        for j, out in enumerate(O.alltoall(ins, "int32")):
            np.testing.assert_array_equal(out, want[j])
        # Broadcast: every rank gets the root's buffer
        for root in {0, p - 1}:
            for out in O.broadcast(ins[root], p, "int32", root):
                np.testing.assert_array_equal(out, ins[root])


@pytest.mark.parametrize("p", PS)
def test_alltoallv_bruteforce(p):
    r = np.random.default_rng(p)
    counts = r.integers(0, 6, size=(p, p))
    counts[r.random((p, p)) < 0.3] = 0
    ins = [r.integers(-50, 50, size=int(counts[i].sum())).astype(np.int32) for i in range(p)]
    outs, rc = O.alltoallv(ins, counts, "int32")
    for j in range(p):
        pieces = []
        for i in range(p):
            parts = np.split(ins[i], np.cumsum(counts[i])[:-1])
            pieces.append(parts[j])
        np.testing.assert_array_equal(outs[j], np.concatenate(pieces))
    np.testing.assert_array_equal(rc, counts.sum(axis=0))
    assert rc.sum() == counts.sum()


def test_alltoallv_rejects_negative_counts():
    with pytest.raises(ValueError):
        O.alltoallv([np.zeros(2, np.int32)] * 2, [[1, -1], [0, 0]], "int32")


# ----------------------------------------------------------------------------------------------
# identities and adjoints stated on the pages

@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("op", ["sum", "min", "max"])
def test_allreduce_equals_allgather_of_reducescatter(p, op):
    n = 12 * p
    for dtype, ins in (("int32", rng_ints(p, p, n)),
                       ("fp32", [x.astype(np.float32) for x in rng_ints(p + 50, p, n)])):
        ar = O.allreduce(ins, dtype, op)
        rs = O.reduce_scatter(ins, dtype, op)
        ag = O.allgather(rs, dtype)
        for r in range(p):
            np.testing.assert_array_equal(ar[r], ag[r])


@pytest.mark.parametrize("p", PS)
def test_allreduce_equals_broadcast_of_reduce(p):
    n = 40
    ins = rng_f32(5 * p, p, n)
    for root in range(p):
        red = O.reduce(ins, "fp32", "sum", root, acc="rankfold")
        bc = O.broadcast(red, p, "fp32", root)
        ar = O.allreduce(ins, "fp32", "sum", acc="rankfold")
        for r in range(p):
            np.testing.assert_array_equal(bc[r], ar[r])


@pytest.mark.parametrize("p", PS)
def test_adjoint_allgather_reducescatter(p):
    m = 9
    r = np.random.default_rng(p)
    x = [r.integers(-100, 100, size=m).astype(np.int32) for _ in range(p)]
    Y = [r.integers(-100, 100, size=p * m).astype(np.int32) for _ in range(p)]
    agx = O.allgather(x, "int32")
    rsy = O.reduce_scatter(Y, "int32", "sum")
    lhs = sum(int(np.dot(agx[q].astype(np.int64), Y[q].astype(np.int64))) for q in range(p))
    rhs = sum(int(np.dot(x[q].astype(np.int64), rsy[q].astype(np.int64))) for q in range(p))
    assert lhs == rhs


@pytest.mark.parametrize("p", PS)
def test_adjoint_broadcast_reduce(p):
    n = 11
    r = np.random.default_rng(10 + p)
    x = r.integers(-100, 100, size=n).astype(np.int32)
    Y = [r.integers(-100, 100, size=n).astype(np.int32) for _ in range(p)]
    for root in range(p):
        bx = O.broadcast(x, p, "int32", root)
        ry = O.reduce(Y, "int32", "sum", root)
        lhs = sum(int(np.dot(bx[q].astype(np.int64), Y[q].astype(np.int64))) for q in range(p))
        assert lhs == int(np.dot(x.astype(np.int64), ry.astype(np.int64)))


@pytest.mark.parametrize("p", PS)
def test_alltoall_twice_is_identity(p):
    ins = rng_ints(p, p, 6 * p)
    back = O.alltoall(O.alltoall(ins, "int32"), "int32")
    for r in range(p):
        np.testing.assert_array_equal(back[r], ins[r])


@pytest.mark.parametrize("p", PS)
def test_alltoallv_transposed_counts_is_inverse(p):
    r = np.random.default_rng(100 + p)
    counts = r.integers(0, 7, size=(p, p))
    ins = [r.integers(-9, 9, size=int(counts[i].sum())).astype(np.int32) for i in range(p)]
    mid, _ = O.alltoallv(ins, counts, "int32")
    back, _ = O.alltoallv(mid, counts.T, "int32")
    for i in range(p):
        np.testing.assert_array_equal(back[i], ins[i])


# ----------------------------------------------------------------------------------------------
# ring schedule emulation

@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("op", ["sum", "min", "max"])
def test_ring_matches_definition_for_exact_types(p, op):
    for n in (0, 1, p - 1 if p > 1 else 1, 5 * p, 5 * p + 3):
        ins = rng_ints(p * 31 + n, p, n, lo=-2**24, hi=2**24)
        direct = O.allreduce(ins, "int32", op)
        for r, out in enumerate(O.ring_allreduce(ins, "int32", op)):
            np.testing.assert_array_equal(out, direct[r])
        for root in range(p):
            np.testing.assert_array_equal(O.ring_reduce(ins, "int32", op, root), direct[0])
        if n % p == 0:
            rs = O.reduce_scatter(ins, "int32", op)
            for r, out in enumerate(O.ring_reduce_scatter(ins, "int32", op)):
                np.testing.assert_array_equal(out, rs[r])
        # integer-valued fp32: every order is exact
        fins = [x.astype(np.float32) for x in rng_ints(p * 37 + n, p, n)]
        exact = O.allreduce(fins, "fp32", op)
        for out in O.ring_allreduce(fins, "fp32", op):
            np.testing.assert_array_equal(out, exact[0])


@pytest.mark.parametrize("p", PS)
def test_ring_fp32_within_error_bound(p):
    n = 64 * p + 5
    ins = rng_f32(p, p, n)
    exact = np.array([math.fsum(float(x[i]) for x in ins) for i in range(n)])
    bound = 2 * p * 2.0**-24 * np.sum(np.abs(np.stack(ins).astype(np.float64)), axis=0)
    for out in O.ring_allreduce(ins, "fp32", "sum"):
        assert np.all(np.abs(out.astype(np.float64) - exact) <= bound)


@pytest.mark.parametrize("p", [2, 3, 4, 5, 8])
def test_ring_fold_order_is_chain_from_next_rank(p):
    """Chunk k is folded as x_{k+1}, ..., x_{p-1}, x_0, ..., x_k (numpy sequential adds)."""
    n = 7 * p
    ins = rng_f32(41 * p, p, n, scale=1e3)
    seg = n // p
    ring = O.ring_allreduce(ins, "fp32", "sum")
    for k in range(p):
        order = [(k + 1 + t) % p for t in range(p)]
        acc = ins[order[0]][k * seg:(k + 1) * seg].copy()
        for q in order[1:]:
            acc = (acc + ins[q][k * seg:(k + 1) * seg]).astype(np.float32)
        for r in range(p):
            np.testing.assert_array_equal(ring[r][k * seg:(k + 1) * seg], acc)


@pytest.mark.parametrize("p", [2, 3, 8])
def test_ring_int32_sum_wraps(p):
    n = 4 * p
    ins = rng_ints(900 + p, p, n, lo=2**30, hi=2**31 - 1)
    want = wrap_i32(np.stack(ins).astype(np.int64).sum(axis=0))
    for out in O.ring_allreduce(ins, "int32", "sum"):
        np.testing.assert_array_equal(out, want)
    np.testing.assert_array_equal(O.ring_reduce(ins, "int32", "sum", p - 1), want)
    for r, out in enumerate(O.ring_reduce_scatter(ins, "int32", "sum")):
        np.testing.assert_array_equal(out, want[r * 4:(r + 1) * 4])


@pytest.mark.parametrize("p", [2, 3, 4, 8])
def test_ring_avg(p):
    # Integer-valued data: every sum is exact in fp32, so the ring's AVG (sum times fl(1/p), rounded
    # once) equals the rank-order AVG; for power-of-two p it equals the exact mean as well.
    n = 16 * p
    ins = [x.astype(np.float32) for x in rng_ints(70 + p, p, n, lo=-1000, hi=1000)]
    want = O.allreduce(ins, "fp32", "avg", acc="rankfold")[0]
    if p & (p - 1) == 0:
        np.testing.assert_array_equal(want, O.allreduce(ins, "fp32", "avg", acc="exact")[0])
    s = O.allreduce(ins, "fp32", "sum", acc="exact")[0]
    assert not np.array_equal(want, s)
    for out in O.ring_allreduce(ins, "fp32", "avg"):
        np.testing.assert_array_equal(out, want)
    for r, out in enumerate(O.ring_reduce_scatter(ins, "fp32", "avg")):
        np.testing.assert_array_equal(out, want[r * 16:(r + 1) * 16])
    np.testing.assert_array_equal(O.ring_reduce(ins, "fp32", "avg", 0), want)
    bins = [bf16_bits_from_f32(x) for x in ins]
    bwant = O.allreduce(bins, "bf16", "avg", acc="rankfold")[0]
    for out in O.ring_allreduce(bins, "bf16", "avg"):
        np.testing.assert_array_equal(out, bwant)


@pytest.mark.parametrize("p", [3, 4, 7])
def test_ring_reduce_chain_order(p):
    n = 33
    ins = rng_f32(43 * p, p, n, scale=1e3)
    for root in range(p):
        order = [(root + 1 + t) % p for t in range(p)]
        acc = ins[order[0]].copy()
        for q in order[1:]:
            acc = (acc + ins[q]).astype(np.float32)
        np.testing.assert_array_equal(O.ring_reduce(ins, "fp32", "sum", root), acc)


@pytest.mark.parametrize("p", PS)
def test_ring_segments_split_evenly_when_p_divides_n(p):
    n = 6 * p
    for k in range(p):
        assert O.ring_segment(n, p, k) == (k * n // p, (k + 1) * n // p)
    # ragged: chunks of ceil(n/p), the last ones shorter; they tile [0, n)
    for n in (1, p + 1, 7 * p - 1):
        segs = [O.ring_segment(n, p, k) for k in range(p)]
        assert segs[0][0] == 0 and segs[-1][1] == n
        assert all(segs[k][1] == segs[k + 1][0] for k in range(p - 1))


# ----------------------------------------------------------------------------------------------
# rounding helpers

def test_float_to_bf16_matches_library_rounding():
    r = np.random.default_rng(0)
    x = np.concatenate([(r.standard_normal(5000) * 10.0 ** r.integers(-30, 30, 5000)).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, 1e-40], np.float32)])
    np.testing.assert_array_equal(O.float_to_bf16(x), bf16_bits_from_f32(x))


def test_double_to_bf16_single_rounding():
    cases = [1.0 + 2.0**-8, 1.0 + 2.0**-8 + 2.0**-40, 1.0 + 3 * 2.0**-8, -(1.0 + 2.0**-8 + 2.0**-40),
             3.0e-39, 2.0**-133 * 0.5 + 2.0**-160, 1e-3, 123456.789]
    r = np.random.default_rng(1)
    cases += list(r.standard_normal(500) * 1e-3)
    got = O.double_to_bf16(cases)
    for c, h in zip(cases, got):
        assert float(bf16_to_f32(np.array([h]))[0]) == exact_round_bf16(Fraction(c)), c
