"""Pins of the oracle's tree AllReduce (single and double binary tree).

Fixed by: the hand-derived fold-order case in golden/tree_fold_order.txt (where the two trees, the
rank-order fold and the exact sum all differ in fp32), exactness on integer-valued data for every
p, brute force for MIN/MAX and int32 wraparound, the power-of-two AVG closed form, p = 1, and bf16
outputs within one ulp of the exact sum.
"""
import os

import numpy as np
import pytest

import oracle
from collective_communication_primitives_b200 import synth as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tree_fold_order.txt")


def _golden():
    g = {"in": {}}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "p":
            g["p"] = int(rest)
        elif key == "in":
            r, _, vals = rest.partition(":")
            g["in"][int(r)] = np.array([float(v) for v in vals.split()], dtype=np.float32)
        else:
            g[key.rstrip(":")] = np.array([float(v) for v in rest.split()], dtype=np.float32)
    return g


def test_tree_fold_order_golden():
    g = _golden()
    ins = [g["in"][r] for r in range(g["p"])]
    for double, key in ((False, "tree_single"), (True, "tree_double")):
        for out in oracle.tree_allreduce(ins, "fp32", "sum", double_tree=double):
            np.testing.assert_array_equal(out, g[key])
    np.testing.assert_array_equal(oracle.allreduce(ins, "fp32", "sum", acc="rankfold")[0], g["rankfold"])
    np.testing.assert_array_equal(oracle.allreduce(ins, "fp32", "sum", acc="exact")[0], g["exact"])


@pytest.mark.parametrize("p", [1, 2, 3, 4, 5, 7, 8, 13, 16])
@pytest.mark.parametrize("double", [False, True])
@pytest.mark.parametrize("n", [1, 2, 7, 64, 129])
def test_integer_data_is_exact(p, double, n):
    ins = [S.ints(f"tree.int.{p}.{r}", n, -1000, 1000).astype(np.float32) for r in range(p)]
    want = np.sum(np.stack(ins).astype(np.float64), axis=0)
    for out in oracle.tree_allreduce(ins, "fp32", "sum", double_tree=double):
        np.testing.assert_array_equal(out.astype(np.float64), want)
    ins_i = [x.astype(np.int32) for x in ins]
    for out in oracle.tree_allreduce(ins_i, "int32", "sum", double_tree=double):
        np.testing.assert_array_equal(out, np.sum(np.stack(ins_i), axis=0, dtype=np.int32))


@pytest.mark.parametrize("p", [2, 3, 6, 8])
@pytest.mark.parametrize("op", ["min", "max"])
@pytest.mark.parametrize("double", [False, True])
def test_min_max_brute_force(p, op, double):
    ins = [S.uniform_pm1(f"tree.mm.{p}.{r}", 50).astype(np.float32) for r in range(p)]
    f = np.min if op == "min" else np.max
    for out in oracle.tree_allreduce(ins, "fp32", op, double_tree=double):
        np.testing.assert_array_equal(out, f(np.stack(ins), axis=0))


def test_int32_wraps():
    big = np.array([2**31 - 1, -2**31], dtype=np.int32)
    ins = [big, big, np.array([5, -5], dtype=np.int32)]
    want = (np.stack(ins).astype(np.int64).sum(axis=0) + 2**31) % 2**32 - 2**31
    for double in (False, True):
        for out in oracle.tree_allreduce(ins, "int32", "sum", double_tree=double):
            np.testing.assert_array_equal(out, want.astype(np.int32))


@pytest.mark.parametrize("p", [2, 4, 8, 16])
def test_avg_power_of_two_is_scaled_sum(p):
    ins = [S.uniform_pm1(f"tree.avg.{p}.{r}", 200).astype(np.float32) for r in range(p)]
    for double in (False, True):
        s = oracle.tree_allreduce(ins, "fp32", "sum", double_tree=double)[0]
        a = oracle.tree_allreduce(ins, "fp32", "avg", double_tree=double)[0]
        np.testing.assert_array_equal(a, (s * np.float32(1.0 / p)).astype(np.float32))


def test_single_rank_is_copy():
    x = S.uniform_pm1("tree.p1", 33).astype(np.float32)
    np.testing.assert_array_equal(oracle.tree_allreduce([x], "fp32", "sum")[0], x)


@pytest.mark.parametrize("double", [False, True])
def test_bf16_within_one_ulp_of_exact(double):
    p, n = 6, 500
    ins = [S.normal(f"tree.bf16.{r}", n, 1.0, "bf16") for r in range(p)]
    got = oracle.bf16_to_float(oracle.tree_allreduce(ins, "bf16", "sum", double_tree=double)[0]).astype(np.float64)
    exact = np.sum(np.stack([oracle.bf16_to_float(x).astype(np.float64) for x in ins]), axis=0)
    ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0**-126))) - 7), 2.0**-133)
    assert (np.abs(got - exact) <= ulp + p * 2.0**-24 * np.sum([np.abs(oracle.bf16_to_float(x)) for x in ins], axis=0)).all()
