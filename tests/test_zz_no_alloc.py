"""The ring AllReduce that allocates nothing (coll_allreduce_ring_noalloc), called through the C ABI.

Some callers cannot allocate device memory (graph capture under a no-allocation policy, allocator
internals, fixed-footprint processes); this entry point runs the ring AllReduce on a static scratch
array inside the library instead of a communicator's scratch. Its results must equal the
communicator's ring AllReduce, on two calls in a row (the scratch keeps the previous call's
contents, so the second call proves that what must start at zero is cleared). This file is
collected last; it creates everything it uses, so it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import check_sum_tolerance, make_inputs, to_numpy, to_torch

pytestmark = pytest.mark.gpu


def c_bufs(sends, recvs):
    p = len(sends)
    s = (ctypes.c_void_p * p)(*[t.data_ptr() for t in sends])
    r = (ctypes.c_void_p * p)(*[t.data_ptr() for t in recvs])
    return SC._Bufs(ctypes.cast(s, ctypes.POINTER(ctypes.c_void_p)),
                    ctypes.cast(r, ctypes.POINTER(ctypes.c_void_p))), (s, r)


@pytest.mark.parametrize("p,n,dtype,op", [(8, 1_000_003, "fp32", "sum"), (8, 700_000, "bf16", "avg"),
                                          (3, 250_001, "int32", "max"), (16, 65_536, "fp32", "avg")])
def test_noalloc_ring_allreduce_matches_the_communicator(p, n, dtype, op):
    L = SC.load_library()
    kind = "int24" if dtype == "int32" else "normal"
    ins = make_inputs(kind, p, n, dtype, f"noalloc.{p}.{n}", sigma=1e-3)
    src = [to_torch(x, dtype) for x in ins]
    want = [torch.empty_like(src[0]) for _ in range(p)]
    with SC.SimComm(p) as c:
        c.allreduce(src, want, op=op, algo="ring")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):  # two calls in a row on the shared static scratch
        got = [torch.full_like(src[0], 7) for _ in range(p)]
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        bufs, keep = c_bufs(src, got)
        rc = L.coll_allreduce_ring_noalloc(p, bufs, n, SC.DTYPES[dtype], SC.OPS[op],
                                           ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(stream))
        assert rc == SC.OK, L.sim_comm_last_error()
        torch.cuda.synchronize()
        assert int(status.item()) == SC.OK
        for r in range(p):
            assert torch.equal(got[r], want[r]), (call, r)
        if dtype != "int32":
            check_sum_tolerance(to_numpy(got[0], dtype), ins, dtype, op, p)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = SC.load_library()
    p, n = 8, 4 << 20  # 8 ranks x 16 MiB of fp32 partials: more than the 32 MiB scratch
    src = [torch.zeros(n, device="cuda") for _ in range(p)]
    dst = [torch.zeros(n, device="cuda") for _ in range(p)]
    bufs, keep = c_bufs(src, dst)
    rc = L.coll_allreduce_ring_noalloc(p, bufs, n, SC.DTYPES["fp32"], SC.OPS["sum"], None,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == SC.INVALID_ARG
    assert b"static scratch" in L.sim_comm_last_error()
    torch.cuda.synchronize()
    assert all(int(torch.count_nonzero(t)) == 0 for t in dst)  # nothing was enqueued
