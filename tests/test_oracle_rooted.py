"""Pins of the rooted copy primitives Scatter and Gather ([Eight] §3.3, §4.3; [Atlas] §0: the
single-root forms of Broadcast/AllGather), through identities with the already pinned ones."""
import numpy as np
import pytest

import oracle as O
from test_oracle_pins import rng_ints

PS = [1, 2, 3, 4, 5, 8]


@pytest.mark.parametrize("p", PS)
def test_scatter_then_allgather_is_broadcast(p):
    for m in (0, 1, 7, 64):
        x = rng_ints(p + m, 1, p * m, lo=-999, hi=999)[0]
        for root in {0, p - 1}:
            parts = O.scatter(x, p, "int32", root)
            for r in range(p):
                np.testing.assert_array_equal(parts[r], x[r * m:(r + 1) * m])  # block r to rank r
            ag = O.allgather(parts, "int32")
            for r, b in enumerate(O.broadcast(x, p, "int32", root)):
                np.testing.assert_array_equal(ag[r], b)


@pytest.mark.parametrize("p", PS)
def test_gather_then_broadcast_is_allgather(p):
    for m in (1, 5, 33):
        shards = rng_ints(7 * p + m, p, m, lo=-999, hi=999)
        for root in range(p):
            g = O.gather(shards, "int32", root)
            np.testing.assert_array_equal(g, np.concatenate(shards))
            for r, (b, a) in enumerate(zip(O.broadcast(g, p, "int32", root), O.allgather(shards, "int32"))):
                np.testing.assert_array_equal(b, a)
            back = O.scatter(g, p, "int32", root)
            for r in range(p):
                np.testing.assert_array_equal(back[r], shards[r])


@pytest.mark.parametrize("p", PS)
def test_scatter_and_gather_are_adjoint(p):
    m = 6
    r = np.random.default_rng(p)
    x = r.integers(-50, 50, size=p * m).astype(np.int32)
    Y = [r.integers(-50, 50, size=m).astype(np.int32) for _ in range(p)]
    for root in range(p):
        sx = O.scatter(x, p, "int32", root)
        gy = O.gather(Y, "int32", root)
        lhs = sum(int(np.dot(sx[q].astype(np.int64), Y[q].astype(np.int64))) for q in range(p))
        assert lhs == int(np.dot(x.astype(np.int64), gy.astype(np.int64)))


def test_rooted_arguments_outside_the_definition():
    with pytest.raises(ValueError):
        O.scatter(np.zeros(7, np.int32), 2, "int32", 0)
    with pytest.raises(ValueError):
        O.gather([np.zeros(2, np.int32)] * 3, "int32", 3)
