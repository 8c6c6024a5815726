"""Full-size workloads on the GPU, checked against the oracle.

Where the oracle can take the whole problem in seconds it does (the DP bucket). Elsewhere the
oracle runs on a sub-selection that commutes with the collective — the same columns of every
row, or the same K positions of every segment, so a ring's segment structure is kept — and
properties that hold at any size are checked on the whole output on the device (replicas equal,
AllReduce == AllGather∘ReduceScatter bit for bit, All-to-All applied twice is the identity, the
combine All-to-Allv restores the input).
"""
import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from collective_communication_primitives_b200 import synth as S
from gpu_helpers import check_sum_tolerance, make_inputs, to_numpy, to_torch

pytestmark = pytest.mark.gpu

M = 1 << 20


def dev(a, dtype):
    return to_torch(a, dtype)


def sample_positions(seg, k, rng):
    """K positions of a segment: its first and last few, and random ones, sorted."""
    edge = [0, 1, 2, seg - 3, seg - 2, seg - 1]
    pos = np.unique(np.concatenate([np.array([x for x in edge if 0 <= x < seg]),
                                    rng.integers(0, seg, size=k)]))
    return pos


def segment_subselection(arrays, p, seg, pos):
    """For each rank, the positions `pos` of every one of its p segments, concatenated, so that the
    reduced problem has p segments of len(pos) elements in the original order."""
    idx = np.concatenate([k * seg + pos for k in range(p)])
    return [a[idx] for a in arrays], idx


# ---- DP gradient bucket: p = 8, 25 Mi elements -------------------------------------------------

@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_dp_bucket_allreduce_avg(dtype, algo):
    p, n = 8, 25 * M
    ins = [S.normal(f"dp.{dtype}.rank{r}", n, 1e-3, dtype) for r in range(p)]
    src = [dev(x, dtype) for x in ins]
    out = [torch.empty_like(src[0]) for _ in range(p)]
    with SC.SimComm(p) as c:
        c.set_option("chunk_bytes", M)
        c.allreduce(src, out, op="avg", algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
    for r in range(1, p):
        assert torch.equal(out[r], out[0])
    got = to_numpy(out[0], dtype)
    want = O.ring_allreduce(ins, dtype, "avg")[0] if algo == "ring" else O.allreduce(ins, dtype, "avg", acc="rankfold")[0]
    np.testing.assert_array_equal(got, want)
    check_sum_tolerance(got, ins, dtype, "avg", p)


# ---- ZeRO shards: p = 8, ReduceScatter of 256 Mi bf16, AllGather of 32 Mi bf16 shards ------------

@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_zero_reduce_scatter_allgather_identity(algo):
    p, n = 8, 256 * M
    m = n // p
    rng = np.random.default_rng(3)
    with SC.SimComm(p) as c:
        c.set_option("chunk_bytes", M)
        grads = [S.normal(f"zero.grad.rank{r}", n, 1e-2, "bf16") for r in range(p)]
        src = [dev(x, "bf16") for x in grads]
        rs = [torch.empty(m, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        c.reduce_scatter(src, rs, op="sum", algo=algo)
        # identity AllReduce == AllGather ∘ ReduceScatter, on the whole tensors, bit for bit
        ag = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        c.allgather(rs, ag, algo=algo)
        ar = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        c.allreduce(src, ar, op="sum", algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        for r in range(p):
            assert torch.equal(ar[r], ag[r]), r
        # sampled ReduceScatter against the oracle on a segment-preserving sub-selection
        pos = sample_positions(m, 4096, rng)
        sub, idx = segment_subselection(grads, p, m, pos)
        want = (O.ring_reduce_scatter(sub, "bf16", "sum") if algo == "ring"
                else O.reduce_scatter(sub, "bf16", "sum", acc="rankfold"))
        pos_t = torch.from_numpy(pos).cuda()
        for r in range(p):
            np.testing.assert_array_equal(to_numpy(rs[r][pos_t], "bf16"), want[r])
        check_sum_tolerance(to_numpy(rs[1][pos_t], "bf16"), [g[m + pos] for g in grads], "bf16", "sum", p)
        del src, ar, ag

        # AllGather of fresh N(0, 0.02) parameter shards
        shards = [S.normal(f"zero.param.rank{r}", m, 0.02, "bf16") for r in range(p)]
        sh = [dev(x, "bf16") for x in shards]
        ag = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        c.allgather(sh, ag, algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
        for r in range(p):
            for q in range(p):
                assert torch.equal(ag[r][q * m:(q + 1) * m], sh[q]), (r, q)
        want = O.allgather([x[pos] for x in shards], "bf16")
        for r in range(p):
            np.testing.assert_array_equal(to_numpy(ag[r][torch.from_numpy(idx).cuda()], "bf16"), want[r])


# ---- MoE dispatch: p = 8, 8,192 tokens x 4,096 bf16 per rank -------------------------------------

@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_moe_alltoall_equal_and_inverse(algo):
    p, tokens, hidden = 8, 8192, 4096
    n = tokens * hidden
    cols = np.sort(np.random.default_rng(4).choice(hidden, 64, replace=False))
    xs = [S.normal(f"moe.x.rank{r}", n, 1.0, "bf16") for r in range(p)]
    with SC.SimComm(p) as c:
        src = [dev(x, "bf16") for x in xs]
        out = [torch.empty_like(src[0]) for _ in range(p)]
        c.alltoall(src, out, algo=algo)
        back = [torch.empty_like(src[0]) for _ in range(p)]
        c.alltoall(out, back, algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
    for r in range(p):
        assert torch.equal(back[r], src[r])
    sub = [x.reshape(tokens, hidden)[:, cols].reshape(-1).copy() for x in xs]
    want = O.alltoall(sub, "bf16")
    cols_t = torch.from_numpy(cols).cuda()
    for r in range(p):
        got = to_numpy(out[r].view(tokens, hidden)[:, cols_t].reshape(-1), "bf16")
        np.testing.assert_array_equal(got, want[r])


@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_moe_alltoallv_dispatch_and_combine(algo):
    p, hidden = 8, 4096
    rows = S.moe_counts(p=p, tokens=8192, experts=64, topk=2, zipf_s=1.1, hidden=1)
    counts = rows * hidden
    send_rows = rows.sum(axis=1)
    assert np.all(send_rows == 16384)
    cap_rows = p * 16384
    cols = np.sort(np.random.default_rng(5).choice(hidden, 48, replace=False))
    xs = [S.normal(f"moe.v.rank{r}", int(send_rows[r]) * hidden, 1.0, "bf16") for r in range(p)]
    with SC.SimComm(p) as c:
        c.set_option("chunk_bytes", M)
        src = [dev(x, "bf16") for x in xs]
        dst = [torch.empty(cap_rows * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        cnt = torch.from_numpy(counts).cuda()
        rc = torch.empty(p, dtype=torch.int64, device="cuda")
        c.alltoallv(src, dst, cnt, algo=algo, recv_counts=rc)
        back = [torch.empty_like(s) for s in src]
        c.alltoallv(dst, back, torch.from_numpy(np.ascontiguousarray(counts.T)).cuda(),
                    recv_cap=[x.numel() for x in back], algo=algo)
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
    np.testing.assert_array_equal(rc.cpu().numpy(), counts.sum(axis=0))
    for r in range(p):
        assert torch.equal(back[r], src[r])
    # oracle on the same 48 columns of every row (counts in rows of 48 elements)
    sub = [x.reshape(-1, hidden)[:, cols].reshape(-1).copy() for x in xs]
    want, _ = O.alltoallv(sub, rows * len(cols), "bf16")
    cols_t = torch.from_numpy(cols).cuda()
    for j in range(p):
        recv_rows = int(rows[:, j].sum())
        got = to_numpy(dst[j][:recv_rows * hidden].view(recv_rows, hidden)[:, cols_t].reshape(-1), "bf16")
        np.testing.assert_array_equal(got, want[j])
    st = S.count_matrix_stats(rows)
    assert st["max_col"] == int(rows.sum(axis=0).max())


# ---- size / rank sweep (bounded: up to 16 MiB per rank in the test) ------------------------------

SWEEP_BYTES = [1 << 10, 1 << 14, 1 << 18, 1 << 22, 1 << 24]


@pytest.mark.parametrize("p", [2, 4, 8, 16, 64])
@pytest.mark.parametrize("algo", ["direct", "ring"])
def test_sweep_int32_exact_and_fp32_bounded(p, algo):
    with SC.SimComm(p) as c:
        c.set_option("chunk_bytes", M)
        for nbytes in SWEEP_BYTES:
            n = max(p, (nbytes // 4) // p * p)
            if p * n > (64 << 20):  # keep the oracle's share of the test to seconds
                continue
            m = n // p
            for dtype, kind, ops in (("int32", "int24", ("sum", "min", "max")), ("fp32", "pm1", ("sum",))):
                ins = make_inputs(kind, p, n, dtype, f"sweep.{p}.{n}")
                src = [dev(x, dtype) for x in ins]
                for op in ops:
                    out = [torch.empty_like(src[0]) for _ in range(p)]
                    c.allreduce(src, out, op=op, algo=algo)
                    rs = [torch.empty(m, dtype=src[0].dtype, device="cuda") for _ in range(p)]
                    c.reduce_scatter(src, rs, op=op, algo=algo)
                    torch.cuda.synchronize()
                    assert c.async_error() == SC.OK
                    if dtype == "int32" or algo == "direct":
                        acc = "exact" if dtype == "int32" else "rankfold"
                        want = O.ring_allreduce(ins, dtype, op) if algo == "ring" else O.allreduce(ins, dtype, op, acc=acc)
                        want_rs = (O.ring_reduce_scatter(ins, dtype, op) if algo == "ring"
                                   else O.reduce_scatter(ins, dtype, op, acc=acc))
                    else:
                        want = O.ring_allreduce(ins, dtype, op)
                        want_rs = O.ring_reduce_scatter(ins, dtype, op)
                    for r in (0, p - 1):
                        np.testing.assert_array_equal(to_numpy(out[r], dtype), want[r])
                        np.testing.assert_array_equal(to_numpy(rs[r], dtype), want_rs[r])
                    for r in range(1, p):
                        assert torch.equal(out[r], out[0])
                    if dtype == "fp32":
                        check_sum_tolerance(to_numpy(out[0], dtype), ins, dtype, "sum", p)
                # copy collectives, bit-exact
                ag = [torch.empty_like(src[0]) for _ in range(p)]
                c.allgather([x[:m] for x in src], ag, algo=algo)
                a2a = [torch.empty_like(src[0]) for _ in range(p)]
                c.alltoall(src, a2a, algo=algo)
                bc = [torch.empty_like(src[0]) for _ in range(p)]
                c.broadcast(src, bc, p // 2, algo=algo)
                torch.cuda.synchronize()
                assert c.async_error() == SC.OK
                want_ag = O.allgather([x[:m] for x in ins], dtype)
                want_a2a = O.alltoall(ins, dtype)
                for r in (0, p // 2, p - 1):
                    np.testing.assert_array_equal(to_numpy(ag[r], dtype), want_ag[r])
                    np.testing.assert_array_equal(to_numpy(a2a[r], dtype), want_a2a[r])
                    np.testing.assert_array_equal(to_numpy(bc[r], dtype), ins[p // 2])
