"""MIN/MAX on data full of signed-zero ties and duplicates, on every reduction schedule, compared bit
for bit with the oracle's emulation of that schedule.

The rule (min(a, b) = b < a ? b : a, max alike, a left fold that keeps the earlier operand on ties)
makes -0.0 and +0.0 distinguishable only by which operand a schedule folds first: the direct path
folds ranks 0..p-1, the ring folds chunk k as x_{k+1}, ..., x_k, the trees fold (own ⊕ left) ⊕
right, the butterflies fold the lower rank first. Integer-valued or Gaussian data never show the
difference (integers give only +0, Gaussians never hit zero), so these inputs are mostly zeros of
random sign: every comparison is made on the raw bits (uint32 for fp32, uint16 for bf16), where
-0.0 and +0.0 differ.
"""
import numpy as np
import pytest

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from collective_communication_primitives_b200 import synth as S
from gpu_helpers import Guarded

pytestmark = pytest.mark.gpu

_COMMS = {}


def comm(p):
    if p not in _COMMS:
        _COMMS[p] = SC.SimComm(p)
    return _COMMS[p]


def tie_inputs(p, n, dtype, label):
    """Per rank: 5/7 zeros, each -0.0 or +0.0 with equal odds, and 1/7 each of -1 and +1."""
    out = []
    for r in range(p):
        v = S.ints(f"{label}.v.rank{r}", n, -3, 3).astype(np.float32)
        neg = S.ints(f"{label}.s.rank{r}", n, 0, 1) == 1
        v[np.abs(v) >= 2] = 0.0
        v = np.where((v == 0) & neg, np.float32(-0.0), v).astype(np.float32)
        out.append(S.fp32_to_bf16_bits(v) if dtype == "bf16" else v)
    return out


def bits(a, dtype):
    return a if dtype == "bf16" else a.view(np.uint32)


def assert_bits_equal(got, want, dtype, what):
    g, w = bits(got, dtype), bits(np.asarray(want), dtype)
    bad = np.flatnonzero(g != w)
    assert bad.size == 0, f"{what}: {bad.size} elements differ, first at {bad[:5]}"


def zero_sign_mix(outs, dtype):
    """Both signs of zero occur among the results (so the case really tests the tie rule)."""
    z = np.concatenate([bits(o, dtype) for o in outs])
    neg_zero = 0x8000 if dtype == "bf16" else 0x80000000
    return bool((z == 0).any() and (z == neg_zero).any())


AR_SCHEDULES = {
    "direct": lambda ins, dt, op: O.allreduce(ins, dt, op),
    "ring": lambda ins, dt, op: O.ring_allreduce(ins, dt, op),
    "ll": lambda ins, dt, op: O.ring_allreduce(ins, dt, op),
    "rd": lambda ins, dt, op: O.rd_allreduce(ins, dt, op),
    "rd_ll": lambda ins, dt, op: O.rd_allreduce(ins, dt, op),
    "hd": lambda ins, dt, op: O.hd_allreduce(ins, dt, op),
    "tree": lambda ins, dt, op: O.tree_allreduce(ins, dt, op),
    "tree_ll": lambda ins, dt, op: O.tree_allreduce(ins, dt, op),
    "dbtree": lambda ins, dt, op: O.tree_allreduce(ins, dt, op, double_tree=True),
    "dbtree_ll": lambda ins, dt, op: O.tree_allreduce(ins, dt, op, double_tree=True),
}


@pytest.mark.parametrize("algo", list(AR_SCHEDULES))
@pytest.mark.parametrize("p", [2, 3, 5, 8])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("op", ["min", "max"])
def test_allreduce_signed_zero_ties(algo, p, dtype, op):
    if algo in ("rd", "rd_ll", "hd") and p & (p - 1):
        pytest.skip("recursive doubling / halving-doubling need p a power of two")
    n = 40_003
    ins = tie_inputs(p, n, dtype, f"ties.ar.{p}")
    c = comm(p)
    src = [Guarded(n, dtype, fill=x) for x in ins]
    out = [Guarded(n, dtype) for _ in range(p)]
    c.allreduce([b.t for b in src], [b.t for b in out], op=op, algo=algo)
    import torch
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    want = AR_SCHEDULES[algo](ins, dtype, op)
    got = [b.numpy() for b in out]
    for r in range(p):
        assert out[r].guards_intact()
        assert_bits_equal(got[r], want[r], dtype, f"{algo} rank {r}")
    assert zero_sign_mix(got, dtype)


@pytest.mark.parametrize("algo", ["direct", "ring"])
@pytest.mark.parametrize("p", [3, 8])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("op", ["min", "max"])
def test_reduce_signed_zero_ties(algo, p, dtype, op):
    n, root = 20_011, 1
    ins = tie_inputs(p, n, dtype, f"ties.red.{p}")
    c = comm(p)
    src = [Guarded(n, dtype, fill=x) for x in ins]
    out = [Guarded(n, dtype) for _ in range(p)]
    c.reduce([b.t for b in src], [b.t for b in out], root, op=op, algo=algo)
    import torch
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    want = O.reduce(ins, dtype, op, root) if algo == "direct" else O.ring_reduce(ins, dtype, op, root)
    got = out[root].numpy()
    assert_bits_equal(got, want, dtype, f"{algo} root")
    assert zero_sign_mix([got], dtype)


@pytest.mark.parametrize("algo", ["direct", "ring", "ll"])
@pytest.mark.parametrize("p", [2, 5, 8])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("op", ["min", "max"])
def test_reduce_scatter_signed_zero_ties(algo, p, dtype, op):
    m = 5_003
    n = p * m
    ins = tie_inputs(p, n, dtype, f"ties.rs.{p}")
    c = comm(p)
    src = [Guarded(n, dtype, fill=x) for x in ins]
    out = [Guarded(m, dtype) for _ in range(p)]
    c.reduce_scatter([b.t for b in src], [b.t for b in out], op=op, algo=algo)
    import torch
    torch.cuda.synchronize()
    assert c.async_error() == SC.OK
    want = O.reduce_scatter(ins, dtype, op) if algo == "direct" else O.ring_reduce_scatter(ins, dtype, op)
    got = [b.numpy() for b in out]
    for r in range(p):
        assert out[r].guards_intact()
        assert_bits_equal(got[r], want[r], dtype, f"{algo} owner {r}")
    assert zero_sign_mix(got, dtype)
