"""Pins of the oracle's MoE dispatch and combine.

What fixes them, besides the oracle itself:
  - the hand-worked example in golden/moe_tiny.txt (count, pack order, receive layout, routing map,
    combine with per-expert scaling and a residual);
  - the definitional properties of the receive layout, checked from the outside on random routes:
    every row sits where the routing map says, sources appear in rank order, rows inside a source
    block are ordered by (expert, token, slot), and every owner holds only its own experts;
  - the reduction to the pinned Alltoallv when k = 1 and the routes are already sorted;
  - closed forms for the combine: round trip with identity experts and weights 1/k, per-expert
    scaling, and the fp32 error bound of the slot-order fold against the exact sum.
"""
import os

import numpy as np
import pytest

import oracle
from collective_communication_primitives_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "moe_tiny.txt")


def _load_golden():
    g = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key in ("p", "T", "k", "H", "E"):
            g[key] = int(rest)
            continue
        if key == "recv_counts:":
            g["recv_counts"] = [int(v) for v in rest.split()]
            continue
        rank, _, vals = rest.partition(":")
        rows = [[float(v) for v in part.split()] for part in vals.split("|")]
        g.setdefault(key, {})[int(rank)] = rows
    return g


def _tiny_inputs(g, dtype):
    xs = [np.array(g["x"][i], dtype=np.float32) for i in range(g["p"])]
    if dtype == "bf16":
        xs = [synth.fp32_to_bf16_bits(x.ravel()).reshape(x.shape) for x in xs]
    elif dtype == "int32":
        xs = [x.astype(np.int32) for x in xs]
    idx = [np.array(g["idx"][i], dtype=np.int32) for i in range(g["p"])]
    w = [np.array(g["w"][i], dtype=np.float32) for i in range(g["p"])]
    return xs, idx, w


def _as_float(a, dtype):
    return oracle.bf16_to_float(a).reshape(a.shape) if dtype == "bf16" else a.astype(np.float64)


@pytest.mark.parametrize("dtype", ["fp32", "bf16", "int32"])
def test_worked_dispatch(dtype):
    g = _load_golden()
    xs, idx, _ = _tiny_inputs(g, dtype)
    res = oracle.moe_dispatch(xs, idx, g["E"], 6, dtype)
    for j in range(g["p"]):
        np.testing.assert_array_equal(_as_float(res["recv"][j], dtype), np.array(g["recv"][j]))
        np.testing.assert_array_equal(res["pos"][j], np.array(g["pos"][j], dtype=np.int32))
        np.testing.assert_array_equal(res["expert_counts"][j], np.array(g["expert_counts"][j][0], dtype=np.int64))
    np.testing.assert_array_equal(res["recv_counts"], np.array(g["recv_counts"]))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("acc", ["exact", "slotfold"])
def test_worked_combine(dtype, acc):
    g = _load_golden()
    xs, idx, w = _tiny_inputs(g, dtype)
    res = oracle.moe_dispatch(xs, idx, g["E"], 6, dtype)
    ys = []
    for j in range(g["p"]):
        scale = 1.0 + np.array(g["recv_expert"][j][0], dtype=np.float32)[:, None]
        yf = (_as_float(res["recv"][j], dtype) * scale).astype(np.float32)
        ys.append(synth.fp32_to_bf16_bits(yf.ravel()).reshape(yf.shape) if dtype == "bf16" else yf)
    ones = np.ones((g["T"], g["H"]), dtype=np.float32)
    resid = [synth.fp32_to_bf16_bits(ones.ravel()).reshape(ones.shape) if dtype == "bf16" else ones] * g["p"]
    outs = oracle.moe_combine(ys, idx, w, dtype, g["E"], residual=resid, acc=acc)
    for i in range(g["p"]):
        np.testing.assert_array_equal(_as_float(outs[i], dtype), np.array(g["combine"][i]))


def _random_case(p, T, k, E, H, seed, dtype="fp32", skew=False):
    rng = np.random.default_rng(seed)
    idx = []
    for _ in range(p):
        if skew:
            ids = np.minimum(rng.geometric(0.35, size=(T, k)) - 1, E - 1)
        else:
            ids = rng.integers(0, E, size=(T, k))
        idx.append(ids.astype(np.int32))
    xs = [rng.integers(-64, 65, size=(T, H)).astype(np.float32) for _ in range(p)]
    if dtype == "bf16":
        xs = [synth.fp32_to_bf16_bits(x.ravel()).reshape(x.shape) for x in xs]
    elif dtype == "int32":
        xs = [x.astype(np.int32) for x in xs]
    return xs, idx


CASES = [(1, 5, 1, 3, 4), (2, 7, 2, 4, 3), (3, 11, 2, 6, 5), (4, 37, 3, 8, 2), (4, 16, 4, 4, 7), (8, 9, 2, 64, 1)]


@pytest.mark.parametrize("p,T,k,E,H", CASES)
@pytest.mark.parametrize("skew", [False, True])
def test_dispatch_layout_properties(p, T, k, E, H, skew):
    xs, idx = _random_case(p, T, k, E, H, seed=p * 100 + T, skew=skew)
    cap = p * T * k
    res = oracle.moe_dispatch(xs, idx, E, cap, "fp32")
    E_loc = E // p
    recv, pos, rc, ec = res["recv"], res["pos"], res["recv_counts"], res["expert_counts"]
    # counts
    for i in range(p):
        np.testing.assert_array_equal(ec[i], np.bincount(idx[i].ravel(), minlength=E))
    c = np.array([[ec[i][j * E_loc:(j + 1) * E_loc].sum() for j in range(p)] for i in range(p)])
    np.testing.assert_array_equal(rc, c.sum(axis=0))
    assert rc.sum() == p * T * k
    # every assignment's row is its token's row, at its expert's owner; the owner's rows are a
    # permutation of [0, rc_j); sources in rank order; (expert, token, slot) increasing inside a block
    seen = [np.zeros(cap, dtype=int) for _ in range(p)]
    for i in range(p):
        for t in range(T):
            for s in range(k):
                e = int(idx[i][t, s])
                j = e // E_loc
                r = int(pos[i][t, s])
                assert 0 <= r < rc[j]
                np.testing.assert_array_equal(recv[j][r], xs[i][t])
                seen[j][r] += 1
                lo = c[:i, j].sum()
                assert lo <= r < lo + c[i, j], "source blocks must follow rank order"
    for j in range(p):
        assert (seen[j][:rc[j]] == 1).all() and (seen[j][rc[j]:] == 0).all()
        np.testing.assert_array_equal(recv[j][rc[j]:], 0)
    for i in range(p):
        keys = sorted((int(pos[i][t, s]), (int(idx[i][t, s]), t, s)) for t in range(T) for s in range(k))
        for j in range(p):
            block = [key for r, key in keys if idx_owner(key[0], E_loc) == j]
            assert block == sorted(block), "a source block must be ordered by (expert, token, slot)"


def idx_owner(e, E_loc):
    return e // E_loc


def test_dispatch_k1_sorted_routes_is_alltoallv():
    p, T, H, E = 4, 10, 3, 8
    rng = np.random.default_rng(7)
    idx = [np.sort(rng.integers(0, E, size=T)).astype(np.int32).reshape(T, 1) for _ in range(p)]
    xs = [rng.integers(-9, 10, size=(T, H)).astype(np.int32) for _ in range(p)]
    res = oracle.moe_dispatch(xs, idx, E, p * T, "int32")
    counts = np.array([[int((idx[i] // (E // p) == j).sum()) * H for j in range(p)] for i in range(p)])
    ref, rc = oracle.alltoallv([x.ravel() for x in xs], counts, "int32")
    for j in range(p):
        np.testing.assert_array_equal(res["recv"][j].ravel()[:ref[j].size], ref[j])
    np.testing.assert_array_equal(res["recv_counts"] * H, rc)


@pytest.mark.parametrize("p,T,k,E,H", [c for c in CASES if c[2] in (1, 2, 4)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("acc", ["exact", "slotfold"])
def test_combine_round_trip_identity(p, T, k, E, H, dtype, acc):
    xs, idx = _random_case(p, T, k, E, H, seed=11 + p, dtype=dtype)
    res = oracle.moe_dispatch(xs, idx, E, p * T * k, dtype)
    w = [np.full((T, k), 1.0 / k, dtype=np.float32) for _ in range(p)]
    outs = oracle.moe_combine(res["recv"], idx, w, dtype, E, acc=acc)
    for i in range(p):
        np.testing.assert_array_equal(outs[i], xs[i])


@pytest.mark.parametrize("p,T,k,E,H", CASES)
def test_combine_per_expert_scaling(p, T, k, E, H):
    """Experts that multiply their rows by (1 + e): out = res + x * Σ_s w_s (1 + e_s), exact for
    small-integer rows and dyadic weights."""
    xs, idx = _random_case(p, T, k, E, H, seed=5 + T)
    res = oracle.moe_dispatch(xs, idx, E, p * T * k, "fp32")
    ys = [r.copy() for r in res["recv"]]
    for i in range(p):
        for t in range(T):
            for s in range(k):
                e = int(idx[i][t, s])
                ys[e // (E // p)][res["pos"][i][t, s]] = xs[i][t] * np.float32(1 + e)
    rng = np.random.default_rng(3)
    w = [(rng.integers(-8, 9, size=(T, k)) / 8.0).astype(np.float32) for _ in range(p)]
    resid = [rng.integers(-5, 6, size=(T, H)).astype(np.float32) for _ in range(p)]
    for acc in ("exact", "slotfold"):
        outs = oracle.moe_combine(ys, idx, w, "fp32", E, residual=resid, acc=acc)
        for i in range(p):
            factor = (w[i].astype(np.float64) * (1.0 + idx[i])).sum(axis=1)
            np.testing.assert_array_equal(outs[i], resid[i] + xs[i] * factor[:, None])


def test_combine_slotfold_error_bound():
    """fp32 fold of k products and a residual: |fold - exact| <= (k+1) 2^-24 (|res| + Σ|w y|)."""
    p, T, k, E, H = 3, 50, 4, 6, 16
    rng = np.random.default_rng(19)
    idx = [rng.integers(0, E, size=(T, k)).astype(np.int32) for _ in range(p)]
    xs = [rng.standard_normal((T, H)).astype(np.float32) for _ in range(p)]
    res = oracle.moe_dispatch(xs, idx, E, p * T * k, "fp32")
    w = [rng.random((T, k)).astype(np.float32) for _ in range(p)]
    resid = [rng.standard_normal((T, H)).astype(np.float32) for _ in range(p)]
    ex = oracle.moe_combine(res["recv"], idx, w, "fp32", E, residual=resid, acc="exact")
    sf = oracle.moe_combine(res["recv"], idx, w, "fp32", E, residual=resid, acc="slotfold")
    for i in range(p):
        mag = np.abs(resid[i]).astype(np.float64) + (np.abs(w[i]).astype(np.float64)[:, :, None] *
                                                       np.abs(xs[i]).astype(np.float64)[:, None, :]).sum(axis=1)
        bound = (k + 1) * 2.0**-24 * mag
        assert (np.abs(sf[i].astype(np.float64) - ex[i].astype(np.float64)) <= bound).all()
        direct = resid[i].astype(np.float64) + (w[i].astype(np.float64)[:, :, None] *
                                                xs[i].astype(np.float64)[:, None, :]).sum(axis=1)
        assert (np.abs(ex[i].astype(np.float64) - direct) <= 2.0**-24 * np.abs(direct) + 1e-30).all()


def test_dispatch_capacity_and_invalid_ids():
    xs, idx = _random_case(2, 6, 2, 4, 3, seed=1)
    need = oracle.moe_dispatch(xs, idx, 4, 24, "fp32")["recv_counts"].max()
    oracle.moe_dispatch(xs, idx, 4, int(need), "fp32")  # exactly enough room
    with pytest.raises(OverflowError):
        oracle.moe_dispatch(xs, idx, 4, int(need) - 1, "fp32")
    bad = [a.copy() for a in idx]
    bad[1][2, 1] = 4
    with pytest.raises(ValueError):
        oracle.moe_dispatch(xs, bad, 4, 24, "fp32")
    with pytest.raises(ValueError):
        oracle.moe_dispatch(xs, idx, 3, 24, "fp32")  # E not a multiple of p


def test_dispatch_empty_tokens():
    xs = [np.zeros((0, 4), dtype=np.float32) for _ in range(3)]
    idx = [np.zeros((0, 2), dtype=np.int32) for _ in range(3)]
    res = oracle.moe_dispatch(xs, idx, 6, 0, "fp32")
    assert res["recv_counts"].sum() == 0
