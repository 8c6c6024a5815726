"""Every communicator entry point refuses an element count, capacity or row count beyond 2^48 with
COLL_ERR_INVALID_ARG before it forms a byte size, so a count whose byte size would wrap around (e.g.
2^62 fp32 elements = 2^64 bytes = 0) can never pass the pointer checks with a false small size.
Nothing is launched: the communicator's launch count stays the same. The pointers are never
dereferenced (the size check comes first), so made-up addresses stand in for buffers."""
import ctypes

import pytest

from collective_communication_primitives_b200 import simcomm as SC

pytestmark = pytest.mark.gpu

HUGE = (1 << 62, (1 << 48) + 4)  # both divisible by p = 4, both above 2^48


def fake_ptrs(p, base):
    arr = (ctypes.c_void_p * p)(*[base + (r << 36) for r in range(p)])
    return arr, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))


@pytest.fixture(scope="module")
def comm():
    c = SC.SimComm(4)
    yield c
    c.close()


def test_collectives_refuse_counts_beyond_2_48(comm):
    L, h, p = SC.load_library(), comm._h, 4
    ks, s = fake_ptrs(p, 0x100000000000)
    kr, r = fake_ptrs(p, 0x500000000000)
    bufs = SC._Bufs(s, r)
    f32 = SC.DTYPES["fp32"]
    before = comm.launch_count()
    for n in HUGE:
        calls = {
            "allreduce": lambda: L.coll_allreduce(h, bufs, n, f32, 0, SC.ALGOS["direct"], None),
            "allreduce ring": lambda: L.coll_allreduce(h, bufs, n, f32, 0, SC.ALGOS["ring"], None),
            "reduce": lambda: L.coll_reduce(h, bufs, n, f32, 0, 1, SC.ALGOS["direct"], None),
            "broadcast": lambda: L.coll_broadcast(h, bufs, n, f32, 1, SC.ALGOS["direct"], None),
            "reduce_scatter": lambda: L.coll_reduce_scatter(h, bufs, n, f32, 0, SC.ALGOS["direct"], None),
            "allgather": lambda: L.coll_allgather(h, bufs, n, f32, SC.ALGOS["direct"], None),
            "alltoall": lambda: L.coll_alltoall(h, bufs, n, f32, SC.ALGOS["direct"], None),
            "scatter": lambda: L.coll_scatter(h, bufs, n, f32, 0, SC.ALGOS["direct"], None),
            "gather": lambda: L.coll_gather(h, bufs, n, f32, 0, SC.ALGOS["direct"], None),
        }
        for name, call in calls.items():
            assert call() == SC.INVALID_ARG, name
            assert b"2^48" in L.sim_comm_last_error(), name
    assert comm.launch_count() == before


def test_alltoallv_refuses_capacities_beyond_2_48(comm):
    L, h, p = SC.load_library(), comm._h, 4
    ks, s = fake_ptrs(p, 0x100000000000)
    kr, r = fake_ptrs(p, 0x500000000000)
    bufs = SC._Bufs(s, r)
    counts = ctypes.c_void_p(0x200000000000)  # 8-byte aligned; never read (refused on the host)
    big = (ctypes.c_longlong * p)(*([1 << 62] * p))
    ok = (ctypes.c_longlong * p)(*([16] * p))
    before = comm.launch_count()
    assert L.coll_alltoallv(h, bufs, counts, big, ok, SC.DTYPES["fp32"], 0, None, None) == SC.INVALID_ARG
    assert b"2^48" in L.sim_comm_last_error()
    assert L.coll_alltoallv(h, bufs, counts, ok, big, SC.DTYPES["fp32"], 0, None, None) == SC.INVALID_ARG
    assert b"2^48" in L.sim_comm_last_error()
    assert comm.launch_count() == before


def test_moe_refuses_rows_times_hidden_beyond_2_48(comm):
    L, h, p = SC.load_library(), comm._h, 4
    kx, x = fake_ptrs(p, 0x100000000000)
    ki, idx = fake_ptrs(p, 0x180000000000)
    ky, y = fake_ptrs(p, 0x500000000000)
    kw, w = fake_ptrs(p, 0x580000000000)
    bf16 = SC.DTYPES["bf16"]
    before = comm.launch_count()
    # tokens x hidden too large
    assert L.coll_moe_dispatch(h, x, idx, 1 << 20, 2, 1 << 30, 8, bf16, y, 16, None, None, None, None) == \
        SC.INVALID_ARG
    # receive capacity x hidden too large
    assert L.coll_moe_dispatch(h, x, idx, 16, 2, 1 << 20, 8, bf16, y, 1 << 30, None, None, None, None) == \
        SC.INVALID_ARG
    # hidden alone beyond 2^48
    assert L.coll_moe_dispatch(h, x, idx, 0, 2, 1 << 62, 8, bf16, y, 0, None, None, None, None) == SC.INVALID_ARG
    # combine: expert-output rows x hidden too large
    assert L.coll_moe_combine(h, y, 1 << 30, idx, idx, w, None, 16, 2, 1 << 20, 8, bf16, x, None) == SC.INVALID_ARG
    assert comm.launch_count() == before
