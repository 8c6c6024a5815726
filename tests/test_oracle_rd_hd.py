"""Pins of the recursive-doubling and halving-doubling AllReduce emulations ([Atlas] §2.3)."""
import math
import os

import numpy as np
import pytest

import oracle as O
from test_oracle_pins import bf16_bits_from_f32, rng_f32, rng_ints, wrap_i32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PS = [1, 2, 4, 8, 16]


def parse(path):
    vals = {}
    for raw in open(path):
        line = raw.split("#")[0].strip()
        if not line:
            continue
        if ":" in line:
            k, v = line.split(":")
            vals[k.strip()] = [float(x) for x in v.split()]
        else:
            k, v = line.split()
            vals[k] = int(v)
    return vals


def test_fold_order_golden():
    g = parse(os.path.join(GOLDEN, "rd_hd_fold_order.txt"))
    ins = [np.array(g[f"in {r}"], np.float32) for r in range(g["p"])]
    assert list(O.allreduce(ins, "fp32", "sum", acc="rankfold")[0]) == g["rank_order"]
    for out in O.rd_allreduce(ins, "fp32", "sum"):
        assert list(out) == g["rd_allreduce"]
    for out in O.hd_allreduce(ins, "fp32", "sum"):
        assert list(out) == g["hd_allreduce"]


@pytest.mark.parametrize("p", PS)
@pytest.mark.parametrize("op", ["sum", "min", "max"])
@pytest.mark.parametrize("algo", ["rd", "hd"])
def test_exact_types_equal_the_definition(p, op, algo):
    f = O.rd_allreduce if algo == "rd" else O.hd_allreduce
    for n in (0, 1, p, 3 * p + 1, 257 * p):
        ins = rng_ints(13 * p + n, p, n, lo=-2**24, hi=2**24)
        stack = np.stack(ins) if n else np.zeros((p, 0), np.int32)
        want = {"sum": lambda: wrap_i32(stack.astype(np.int64).sum(axis=0)),
                "min": lambda: stack.min(axis=0), "max": lambda: stack.max(axis=0)}[op]()
        for out in f(ins, "int32", op):
            np.testing.assert_array_equal(out, want)
        fins = [x.astype(np.float32) for x in rng_ints(17 * p + n, p, n)]
        exact = O.allreduce(fins, "fp32", op)[0]
        for out in f(fins, "fp32", op):
            np.testing.assert_array_equal(out, exact)


@pytest.mark.parametrize("p", [2, 4, 8, 16])
@pytest.mark.parametrize("algo", ["rd", "hd"])
def test_fp32_and_bf16_bounds_and_identical_replicas(p, algo):
    f = O.rd_allreduce if algo == "rd" else O.hd_allreduce
    n = 33 * p + 5
    ins = rng_f32(21 * p, p, n)
    exact = np.array([math.fsum(float(x[i]) for x in ins) for i in range(n)])
    bound = 2 * p * 2.0**-24 * np.sum(np.abs(np.stack(ins).astype(np.float64)), axis=0)
    outs = f(ins, "fp32", "sum")
    for out in outs:
        np.testing.assert_array_equal(out, outs[0])
        assert np.all(np.abs(out.astype(np.float64) - exact) <= bound)
    b = [bf16_bits_from_f32(x) for x in ins]
    for out in f(b, "bf16", "avg"):
        assert out.dtype == np.uint16


def test_recursive_doubling_is_a_balanced_tree_fold():
    """p = 8, recursive doubling folds ((x0+x1)+(x2+x3))+((x4+x5)+(x6+x7)) (numpy adds)."""
    p, n = 8, 64
    ins = rng_f32(99, p, n, scale=1e4)
    t = [(ins[2 * i] + ins[2 * i + 1]).astype(np.float32) for i in range(4)]
    t = [(t[0] + t[1]).astype(np.float32), (t[2] + t[3]).astype(np.float32)]
    want = (t[0] + t[1]).astype(np.float32)
    for out in O.rd_allreduce(ins, "fp32", "sum"):
        np.testing.assert_array_equal(out, want)


def test_non_power_of_two_is_rejected():
    with pytest.raises(ValueError):
        O.rd_allreduce([np.zeros(3, np.float32)] * 3, "fp32", "sum")
    with pytest.raises(ValueError):
        O.hd_allreduce([np.zeros(3, np.float32)] * 6, "fp32", "sum")
