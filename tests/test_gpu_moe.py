"""GPU parity of the MoE dispatch and combine (C-ABI library) against the oracle.

Dispatch is a copy plus integer bookkeeping, so everything is bit-exact: the received rows, the
untouched rows past each receive count, the routing map and both count outputs. The combine is
bit-exact against the oracle's fp32 slot-order fold, and within the fold's error bound of the exact
(double) sum. The MoE workload at full size (8 ranks x 8192 tokens, top-2 of 64 experts, Zipf(1.1)
routes, 4096-wide bf16 rows) is checked through the exact routing map (oracle on token ids), a
device-side check of every received row, and oracle recomputation of sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from collective_communication_primitives_b200 import simcomm as SC
from collective_communication_primitives_b200 import synth as S
from gpu_helpers import SENT, Guarded, to_numpy, to_torch

pytestmark = pytest.mark.gpu


def make_routes(p, T, k, E, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        ids = rng.integers(0, E, size=(p, T, k))
    elif kind == "skew":
        ids = np.minimum(rng.geometric(0.3, size=(p, T, k)) - 1, E - 1)
    elif kind == "one":
        ids = np.full((p, T, k), E - 1)
    elif kind == "zipf":
        ids = S.moe_routes(p, T, E, k, 1.1, seed)
    else:
        raise ValueError(kind)
    return ids.astype(np.int32)


def make_rows(p, T, H, dtype, label):
    out = []
    for i in range(p):
        if dtype == "int32":
            v = S.ints(f"{label}.rank{i}", T * H, -2**24, 2**24).astype(np.int32)
        else:
            v = S.normal(f"{label}.rank{i}", T * H, 1.0, dtype)
        out.append(v.reshape(T, H))
    return out


def rows2d(g, H):
    return g.t.view(-1, H)


def dispatch_case(comm, xs, ids, E, cap, dtype, offset=0):
    p = len(xs)
    T, k = ids[0].shape
    H = xs[0].shape[1]
    x_g = [Guarded(T * H, dtype, offset, fill=x.ravel()) for x in xs]
    r_g = [Guarded(cap * H, dtype, offset) for _ in range(p)]
    idx_t = [to_torch(a.ravel(), "int32").view(T, k) for a in ids]
    pos_t = [torch.full((T, k), -7, dtype=torch.int32, device="cuda") for _ in range(p)]
    ec = torch.full((p, E), -1, dtype=torch.int64, device="cuda")
    rc = torch.full((p,), -1, dtype=torch.int64, device="cuda")
    comm.moe_dispatch([rows2d(g, H) for g in x_g], idx_t, E, [rows2d(g, H) for g in r_g], route_pos=pos_t,
                      expert_counts=ec, recv_counts=rc)
    torch.cuda.synchronize()
    return x_g, r_g, idx_t, pos_t, ec, rc


DISPATCH_CASES = [
    # p, T, k, E, H, dtype, routes, element offset of every buffer
    (1, 40, 2, 4, 8, "fp32", "uniform", 0),
    (2, 300, 2, 4, 24, "bf16", "skew", 0),
    (3, 257, 1, 6, 7, "fp32", "uniform", 0),
    (4, 520, 3, 8, 16, "bf16", "skew", 0),
    (4, 130, 2, 4, 64, "int32", "one", 0),
    (8, 1000, 2, 64, 128, "bf16", "zipf", 0),
    (8, 600, 4, 16, 40, "fp32", "uniform", 1),
    (5, 77, 2, 5, 33, "bf16", "skew", 0),
    (16, 64, 2, 32, 8, "fp32", "uniform", 0),
    (64, 8, 2, 64, 4, "int32", "uniform", 0),
    (2, 4000, 8, 256, 12, "fp32", "uniform", 0),
    (3, 50, 2, 6, 5000, "bf16", "skew", 0),     # 10,000-byte rows: two bulk tiles per row
    (2, 40, 3, 4, 4100, "fp32", "uniform", 0),  # 16,400-byte rows: three bulk tiles, a short last one
]


@pytest.mark.parametrize("p,T,k,E,H,dtype,kind,offset", DISPATCH_CASES)
@pytest.mark.parametrize("fused,tma", [(1, 0), (0, 1), (0, 0)])
def test_dispatch_parity(p, T, k, E, H, dtype, kind, offset, fused, tma):
    """Every dispatch path: the fused cooperative kernel (32/16/2-byte copies), and the three-kernel
    path with either copy kernel: bulk copies through shared memory (rows of whole 16-byte units at
    aligned bases, else the load/store kernel runs) and 32/16/2-byte loads and stores."""
    ids = make_routes(p, T, k, E, kind, seed=p * 31 + T)
    xs = make_rows(p, T, H, dtype, f"moe.dispatch.{p}.{T}.{H}")
    ref = oracle.moe_dispatch(xs, list(ids), E, p * T * k, dtype)
    cap = int(ref["recv_counts"].max()) + 3
    with SC.SimComm(p) as comm:
        comm.set_option("moe_fused", fused)
        comm.set_option("moe_tma", tma)
        x_g, r_g, _, pos_t, ec, rc = dispatch_case(comm, xs, ids, E, cap, dtype, offset)
        assert comm.async_error() == SC.OK
    np.testing.assert_array_equal(rc.cpu().numpy(), ref["recv_counts"])
    np.testing.assert_array_equal(ec.cpu().numpy(), ref["expert_counts"])
    for i in range(p):
        np.testing.assert_array_equal(pos_t[i].cpu().numpy(), ref["pos"][i])
        np.testing.assert_array_equal(x_g[i].numpy().reshape(T, H), xs[i])
    for j in range(p):
        got = r_g[j].numpy().reshape(cap, H)
        n = int(ref["recv_counts"][j])
        np.testing.assert_array_equal(got[:n], ref["recv"][j][:n])
        assert (got[n:] == SENT[dtype]).all(), "rows past the received count must stay untouched"
        assert r_g[j].guards_intact()


SHAPE_SEQUENCE = [
    # p, T, k, E, H, dtype, routes: one communicator, in this order
    (4, 4000, 4, 16, 8, "bf16", "zipf"),     # 63 counting tiles per rank: up to two earlier-tile loads per lane
    (4, 300, 2, 8, 16, "fp32", "skew"),      # fewer experts: the totals array is partly reused
    (4, 5000, 4, 16, 8, "bf16", "uniform"),  # 79 tiles per rank: the long path (prefix phase)
    (4, 1000, 2, 4096, 4, "fp32", "uniform"),  # first-row table too large for shared memory
    (4, 4000, 4, 16, 8, "bf16", "zipf"),     # the short path again, after both long forms
    (2, 1500, 8, 64, 4, "int32", "skew"),    # short path, 8 slots per token: 16 lookups per batch
    (2, 600, 4, 2048, 8, "fp32", "uniform"), # short path with more experts than per-warp histograms hold
    (2, 3000, 8, 64, 4, "int32", "skew"),    # 94 tiles per rank: long path, 8 slots per token
]


def test_fused_dispatch_shape_sequence_on_one_communicator():
    """The fused dispatch keeps per-(rank, expert) totals between calls only as zeros: its short path
    (at most 64 counting tiles per rank and a first-row table in shared memory) sums them during
    counting and its last CTA clears them. Calls of changing shape on one communicator, short and long
    paths interleaved, each bit-exact against the oracle; then an overflow (which leaves the totals
    uncleared), a reset, and a short-path call that must again match."""
    comm = SC.SimComm(SHAPE_SEQUENCE[0][0])
    try:
        for case_no, (p, T, k, E, H, dtype, kind) in enumerate(SHAPE_SEQUENCE):
            if p != comm.p:  # a new communicator only where the rank count changes
                comm.close()
                comm = SC.SimComm(p)
            ids = make_routes(p, T, k, E, kind, seed=100 + case_no)
            xs = make_rows(p, T, H, dtype, f"moe.seq.{case_no}")
            ref = oracle.moe_dispatch(xs, list(ids), E, p * T * k, dtype)
            cap = int(ref["recv_counts"].max())
            _, r_g, _, pos_t, ec, rc = dispatch_case(comm, xs, ids, E, cap, dtype)
            assert comm.async_error() == SC.OK, case_no
            np.testing.assert_array_equal(rc.cpu().numpy(), ref["recv_counts"], err_msg=str(case_no))
            np.testing.assert_array_equal(ec.cpu().numpy(), ref["expert_counts"], err_msg=str(case_no))
            for i in range(p):
                np.testing.assert_array_equal(pos_t[i].cpu().numpy(), ref["pos"][i], err_msg=str(case_no))
            for j in range(p):
                n = int(ref["recv_counts"][j])
                np.testing.assert_array_equal(r_g[j].numpy().reshape(cap, H)[:n], ref["recv"][j][:n],
                                              err_msg=str(case_no))
    finally:
        comm.close()
    p, T, k, E, H, dtype, kind = SHAPE_SEQUENCE[0]
    ids = make_routes(p, T, k, E, kind, seed=100)
    xs = make_rows(p, T, H, dtype, "moe.seq.0")
    ref = oracle.moe_dispatch(xs, list(ids), E, p * T * k, dtype)
    with SC.SimComm(p) as comm:
        _, r_g, _, _, _, _ = dispatch_case(comm, xs, ids, E, int(ref["recv_counts"].max()) - 1, dtype)
        assert comm.async_error() == SC.OVERFLOW
        comm.reset()
        cap = int(ref["recv_counts"].max())
        _, r_g, _, pos_t, ec, rc = dispatch_case(comm, xs, ids, E, cap, dtype)
        assert comm.async_error() == SC.OK
        np.testing.assert_array_equal(ec.cpu().numpy(), ref["expert_counts"])
        for i in range(p):
            np.testing.assert_array_equal(pos_t[i].cpu().numpy(), ref["pos"][i])
        for j in range(p):
            n = int(ref["recv_counts"][j])
            np.testing.assert_array_equal(r_g[j].numpy().reshape(cap, H)[:n], ref["recv"][j][:n])


def combine_inputs(p, T, k, cap, H, dtype, seed):
    ys = make_rows(p, cap, H, dtype, f"moe.y.{seed}")
    w = S.moe_gate_weights(p, T, k, seed)
    res = make_rows(p, T, H, dtype, f"moe.res.{seed}")
    return ys, [w[i] for i in range(p)], res


@pytest.mark.parametrize("p,T,k,E,H,dtype,kind,offset", [c for c in DISPATCH_CASES if c[5] != "int32"])
@pytest.mark.parametrize("residual", ["none", "separate", "inplace"])
def test_combine_parity(p, T, k, E, H, dtype, kind, offset, residual):
    ids = make_routes(p, T, k, E, kind, seed=p * 17 + T)
    ref = oracle.moe_dispatch([np.zeros((T, 1), np.int32)] * p, list(ids), E, p * T * k, "int32")
    cap = int(ref["recv_counts"].max()) + 1
    ys, ws, res = combine_inputs(p, T, k, cap, H, dtype, seed=T + k)
    want = oracle.moe_combine(ys, list(ids), ws, dtype, E, residual=None if residual == "none" else res,
                              acc="slotfold")
    exact = oracle.moe_combine(ys, list(ids), ws, dtype, E, residual=None if residual == "none" else res,
                               acc="exact")
    y_g = [Guarded(cap * H, dtype, offset, fill=y.ravel()) for y in ys]
    o_g = [Guarded(T * H, dtype, offset, fill=(r.ravel() if residual == "inplace" else None)) for r in res]
    r_t = None
    if residual == "separate":
        r_t = [to_torch(r.ravel(), dtype).view(T, H) for r in res]
    elif residual == "inplace":
        r_t = [rows2d(g, H) for g in o_g]
    idx_t = [to_torch(a.ravel(), "int32").view(T, k) for a in ids]
    pos_t = [to_torch(a.ravel(), "int32").view(T, k) for a in ref["pos"]]
    w_t = [to_torch(w.ravel(), "fp32").view(T, k) for w in ws]
    with SC.SimComm(p) as comm:
        comm.moe_combine([rows2d(g, H) for g in y_g], idx_t, pos_t, w_t, E, [rows2d(g, H) for g in o_g],
                         residual=r_t)
        torch.cuda.synchronize()
        assert comm.async_error() == SC.OK
    for i in range(p):
        got = o_g[i].numpy().reshape(T, H)
        np.testing.assert_array_equal(got, want[i])
        assert o_g[i].guards_intact()
        if dtype == "fp32":
            mag = np.abs(res[i]).astype(np.float64) if residual != "none" else 0.0
            e = ids[i] // (E // p)
            rows = np.stack([ys[e[:, s][t]][ref["pos"][i][t, s]] for t in range(T) for s in range(k)]).reshape(T, k, H)
            mag = mag + (np.abs(ws[i]).astype(np.float64)[:, :, None] * np.abs(rows).astype(np.float64)).sum(axis=1)
            err = np.abs(got.astype(np.float64) - exact[i].astype(np.float64))
            assert (err <= (k + 1) * 2.0**-24 * mag + 1e-38).all()


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_round_trip_identity_experts(dtype):
    """dispatch -> identity experts -> combine with weights 1/2 returns the tokens bit for bit."""
    p, T, k, E, H = 4, 700, 2, 16, 96
    ids = make_routes(p, T, k, E, "skew", seed=3)
    xs = make_rows(p, T, H, dtype, "moe.roundtrip")
    with SC.SimComm(p) as comm:
        x_g, r_g, idx_t, pos_t, _, _ = dispatch_case(comm, xs, ids, E, p * T * k, dtype)
        w_t = [torch.full((T, k), 0.5, dtype=torch.float32, device="cuda") for _ in range(p)]
        out = [torch.empty(T, H, dtype=x_g[0].t.dtype, device="cuda") for _ in range(p)]
        comm.moe_combine([rows2d(g, H) for g in r_g], idx_t, pos_t, w_t, E, out)
        torch.cuda.synchronize()
        assert comm.async_error() == SC.OK
    for i in range(p):
        np.testing.assert_array_equal(to_numpy(out[i], dtype), xs[i])


def test_full_size_moe_workload():
    """8 ranks x 8192 tokens, top-2 of 64 experts, Zipf(1.1) routes, 4096-wide bf16 rows."""
    p, T, k, E, H, dtype = 8, 8192, 2, 64, 4096, "bf16"
    cap = p * T * k  # every assignment could go to one rank
    ids = S.moe_routes(p, T, E, k, 1.1, 0)
    ref = oracle.moe_dispatch([np.arange(T, dtype=np.int32).reshape(T, 1) + i * T for i in range(p)], list(ids), E,
                              cap, "int32")
    xs = [torch.from_numpy(S.normal(f"moe.full.x.rank{i}", T * H, 1.0, "bf16").view(np.int16)).view(torch.bfloat16)
          .cuda().view(T, H) for i in range(p)]
    recv = [torch.full((cap, H), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    idx_t = [torch.from_numpy(ids[i]).cuda() for i in range(p)]
    pos_t = [torch.empty(T, k, dtype=torch.int32, device="cuda") for _ in range(p)]
    ec = torch.empty(p, E, dtype=torch.int64, device="cuda")
    rc = torch.empty(p, dtype=torch.int64, device="cuda")
    with SC.SimComm(p) as comm:
        comm.moe_dispatch(xs, idx_t, E, recv, route_pos=pos_t, expert_counts=ec, recv_counts=rc)
        torch.cuda.synchronize()
        assert comm.async_error() == SC.OK
        np.testing.assert_array_equal(rc.cpu().numpy(), ref["recv_counts"])
        np.testing.assert_array_equal(ec.cpu().numpy(), ref["expert_counts"])
        owner = [torch.from_numpy(ids[i] // (E // p)).cuda().long() for i in range(p)]
        for i in range(p):
            np.testing.assert_array_equal(pos_t[i].cpu().numpy(), ref["pos"][i])
            # every assignment's received row is its token's row (the map is exact, so this covers
            # every received row)
            for j in range(p):
                sel = owner[i] == j
                tok = torch.nonzero(sel)[:, 0]
                rows = pos_t[i][sel].long()
                assert torch.equal(recv[j].index_select(0, rows).view(torch.int16),
                                   xs[i].index_select(0, tok).view(torch.int16))
        for j in range(p):
            n = int(ref["recv_counts"][j])
            assert torch.isnan(recv[j][n:].float()).all(), "rows past the received count must stay untouched"

        # combine: identity experts (y = recv), synthetic gate weights and residual
        ws = S.moe_gate_weights(p, T, k, 0)
        w_t = [torch.from_numpy(ws[i]).cuda() for i in range(p)]
        res_np = [S.normal(f"moe.full.res.rank{i}", T * H, 1.0, "bf16").reshape(T, H) for i in range(p)]
        res_t = [to_torch(r.ravel(), "bf16").view(T, H) for r in res_np]
        out = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        comm.moe_combine(recv, idx_t, pos_t, w_t, E, out, residual=res_t)
        torch.cuda.synchronize()
        assert comm.async_error() == SC.OK
    # sampled tokens, recomputed by the oracle on a reduced problem with the same rows
    rng = np.random.default_rng(0)
    Ts = 48
    samp = [np.sort(rng.choice(T, Ts, replace=False)) for _ in range(p)]
    ids_s = [ids[i][samp[i]] for i in range(p)]
    ref_s = oracle.moe_dispatch([np.zeros((Ts, 1), np.int32)] * p, ids_s, E, p * Ts * k, "int32")
    y_s = [np.zeros((p * Ts * k, H), dtype=np.uint16) for _ in range(p)]
    for i in range(p):
        for a, t in enumerate(samp[i]):
            for s in range(k):
                j = int(ids[i][t, s]) // (E // p)
                y_s[j][ref_s["pos"][i][a, s]] = to_numpy(recv[j][int(ref["pos"][i][t, s])], "bf16")
    want = oracle.moe_combine(y_s, ids_s, [ws[i][samp[i]] for i in range(p)], "bf16", E,
                              residual=[res_np[i][samp[i]] for i in range(p)], acc="slotfold")
    for i in range(p):
        got = to_numpy(out[i], "bf16")[samp[i]]
        np.testing.assert_array_equal(got, want[i])


@pytest.mark.parametrize("p,T,k,E,H", [(64, 40, 32, 4096, 8), (64, 3, 1, 64, 2), (8, 1, 32, 4096, 16)])
def test_dispatch_and_combine_at_the_limits(p, T, k, E, H):
    """The largest shapes the interface accepts: 64 ranks, 32 slots per token, 4,096 experts."""
    ids = make_routes(p, T, k, E, "uniform", seed=E + k)
    xs = make_rows(p, T, H, "fp32", f"moe.limits.{p}.{k}.{E}")
    ref = oracle.moe_dispatch(xs, list(ids), E, p * T * k, "fp32")
    cap = int(ref["recv_counts"].max())
    with SC.SimComm(p) as comm:
        x_g, r_g, idx_t, pos_t, ec, rc = dispatch_case(comm, xs, ids, E, cap, "fp32")
        assert comm.async_error() == SC.OK
        np.testing.assert_array_equal(ec.cpu().numpy(), ref["expert_counts"])
        for i in range(p):
            np.testing.assert_array_equal(pos_t[i].cpu().numpy(), ref["pos"][i])
        for j in range(p):
            n = int(ref["recv_counts"][j])
            np.testing.assert_array_equal(r_g[j].numpy().reshape(cap, H)[:n], ref["recv"][j][:n])
        ws = S.moe_gate_weights(p, T, k, 1)
        w_t = [to_torch(w.ravel(), "fp32").view(T, k) for w in ws]
        out = [torch.empty(T, H, device="cuda") for _ in range(p)]
        comm.moe_combine([rows2d(g, H) for g in r_g], idx_t, pos_t, w_t, E, out)
        torch.cuda.synchronize()
        assert comm.async_error() == SC.OK
    want = oracle.moe_combine([r[:cap] for r in ref["recv"]], list(ids), list(ws), "fp32", E, acc="slotfold")
    for i in range(p):
        np.testing.assert_array_equal(out[i].cpu().numpy(), want[i])


@pytest.mark.parametrize("fused", [1, 0])
def test_dispatch_overflow_and_invalid_ids_copy_nothing(fused):
    p, T, k, E, H, dtype = 4, 200, 2, 8, 16, "fp32"
    ids = make_routes(p, T, k, E, "one", seed=1)
    xs = make_rows(p, T, H, dtype, "moe.err")
    need = p * T * k
    with SC.SimComm(p) as comm:
        comm.set_option("moe_fused", fused)
        _, r_g, _, _, _, _ = dispatch_case(comm, xs, ids, E, need - 1, dtype)
        assert comm.async_error() == SC.OVERFLOW
        for g in r_g:
            assert (g.numpy() == SENT[dtype]).all()
        comm.reset()
        _, r_g, _, _, _, rc = dispatch_case(comm, xs, ids, E, need, dtype)
        assert comm.async_error() == SC.OK
        assert int(rc[-1]) == need
        bad = ids.copy()
        bad[2, 17, 1] = E
        _, r_g, _, _, _, _ = dispatch_case(comm, xs, bad, E, need, dtype)
        assert comm.async_error() == SC.INVALID_ARG
        for g in r_g:
            assert (g.numpy() == SENT[dtype]).all()
        comm.reset()


def test_combine_rejects_bad_route():
    p, T, k, E, H = 2, 50, 2, 4, 8
    with SC.SimComm(p) as comm:
        y = [torch.zeros(10, H, device="cuda") for _ in range(p)]
        idx = [torch.zeros(T, k, dtype=torch.int32, device="cuda") for _ in range(p)]
        pos = [torch.zeros(T, k, dtype=torch.int32, device="cuda") for _ in range(p)]
        pos[1][3, 1] = 10  # past the 10 rows of y
        w = [torch.ones(T, k, device="cuda") for _ in range(p)]
        out = [torch.zeros(T, H, device="cuda") for _ in range(p)]
        comm.moe_combine(y, idx, pos, w, E, out)
        torch.cuda.synchronize()
        assert comm.async_error() == SC.INVALID_ARG
        comm.reset()


def test_sync_argument_errors_and_empty():
    p, T, k, E, H = 4, 16, 2, 8, 4
    with SC.SimComm(p) as comm:
        x = [torch.zeros(T, H, device="cuda") for _ in range(p)]
        idx = [torch.zeros(T, k, dtype=torch.int32, device="cuda") for _ in range(p)]
        recv = [torch.zeros(p * T * k, H, device="cuda") for _ in range(p)]
        for bad_E in (6, 2, 4097 * p):
            with pytest.raises(SC.SimCommError) as ei:
                comm.moe_dispatch(x, idx, bad_E, recv)
            assert ei.value.status == SC.INVALID_ARG
        with pytest.raises(SC.SimCommError) as ei:
            comm.moe_dispatch(x, idx, E, [x[0]] + recv[1:])  # an output overlapping an input
        assert ei.value.status == SC.INVALID_ARG
        with pytest.raises(SC.SimCommError) as ei:
            comm.moe_combine([r.int() for r in recv], idx, idx, [torch.ones(T, k, device="cuda")] * p, E,
                             [torch.zeros(T, H, dtype=torch.int32, device="cuda") for _ in range(p)])
        assert ei.value.status == SC.UNSUPPORTED
        big = [torch.zeros(T, 33, dtype=torch.int32, device="cuda") for _ in range(p)]
        with pytest.raises(SC.SimCommError) as ei:
            comm.moe_dispatch(x, big, E, recv)  # k = 33
        assert ei.value.status == SC.INVALID_ARG
        # no tokens: only the counts change
        ec = torch.full((p, E), 5, dtype=torch.int64, device="cuda")
        rc = torch.full((p,), 5, dtype=torch.int64, device="cuda")
        comm.moe_dispatch([t[:0] for t in x], [t[:0] for t in idx], E, recv, expert_counts=ec, recv_counts=rc)
        torch.cuda.synchronize()
        assert int(ec.abs().sum()) == 0 and int(rc.abs().sum()) == 0
        assert comm.async_error() == SC.OK
