"""The ring AllReduce that allocates nothing (coll_allreduce_ring_noalloc), called through the C ABI.

Some callers cannot allocate device memory: an allocator or memory pool (it must not re-enter the
allocator it implements), a process whose device footprint is fixed at start-up, or code where a
framework forbids allocation. This entry point runs the ring AllReduce on a static scratch array
inside the library instead of a communicator's scratch. Its results must equal the oracle's ring
emulation bit for bit and the communicator's ring AllReduce, on two calls in a row (the scratch keeps
the previous call's contents, so the second call proves that what must start at zero is cleared).

This file is collected last. It creates everything it uses, so it also passes alone in a fresh
process; one case runs the entry point as the very first library call of a child process that never
creates a communicator.
"""
import ctypes
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle as O
from collective_communication_primitives_b200 import simcomm as SC
from gpu_helpers import check_sum_tolerance, make_inputs, to_numpy, to_torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def c_bufs(sends, recvs):
    p = len(sends)
    s = (ctypes.c_void_p * p)(*[t.data_ptr() for t in sends])
    r = (ctypes.c_void_p * p)(*[t.data_ptr() for t in recvs])
    return SC._Bufs(ctypes.cast(s, ctypes.POINTER(ctypes.c_void_p)),
                    ctypes.cast(r, ctypes.POINTER(ctypes.c_void_p))), (s, r)


def noalloc(L, src, got, n, dtype, op, status):
    bufs, keep = c_bufs(src, got)
    rc = L.coll_allreduce_ring_noalloc(len(src), bufs, n, SC.DTYPES[dtype], SC.OPS[op],
                                       ctypes.c_void_p(status.data_ptr()),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == SC.OK, L.sim_comm_last_error()


def bits(a):
    return a.view(np.uint32) if a.dtype == np.float32 else a  # tells -0.0 from +0.0


@pytest.mark.parametrize("p,n,dtype,op", [(8, 1_000_003, "fp32", "sum"), (8, 700_000, "bf16", "avg"),
                                          (3, 250_001, "int32", "max"), (16, 65_536, "fp32", "avg"),
                                          (5, 4_099, "fp32", "min"), (2, 1, "bf16", "sum")])
def test_noalloc_ring_allreduce_matches_oracle_and_communicator(p, n, dtype, op):
    L = SC.load_library()
    kind = "int24" if dtype == "int32" else "normal"
    ins = make_inputs(kind, p, n, dtype, f"noalloc.{p}.{n}", sigma=1e-3)
    oracle = O.ring_allreduce(ins, dtype, op)
    src = [to_torch(x, dtype) for x in ins]
    comm_out = [torch.empty_like(src[0]) for _ in range(p)]
    with SC.SimComm(p) as c:
        c.allreduce(src, comm_out, op=op, algo="ring")
        torch.cuda.synchronize()
        assert c.async_error() == SC.OK
    for call in range(2):  # two calls in a row on the shared static scratch
        got = [torch.full_like(src[0], 7) for _ in range(p)]
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        noalloc(L, src, got, n, dtype, op, status)
        torch.cuda.synchronize()
        assert int(status.item()) == SC.OK
        for r in range(p):
            g = to_numpy(got[r], dtype)
            np.testing.assert_array_equal(bits(g), bits(oracle[r]), err_msg=f"call {call} rank {r} vs oracle")
            assert torch.equal(got[r], comm_out[r]), (call, r)
        if dtype != "int32" and op in ("sum", "avg"):
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


def test_noalloc_timeout_status_then_recovers():
    """Host-side fault injection: rank 1 never signals, so its successor's bounded wait runs out after
    the 50 ms timeout and the call reports COLL_ERR_TIMEOUT through async_status_dev; the next call,
    with injection off, clears the shared scratch and gives the oracle's result again."""
    L = SC.load_library()
    p, n, dtype, op = 4, 40_000, "fp32", "sum"
    ins = make_inputs("normal", p, n, dtype, "noalloc.timeout", sigma=1e-3)
    src = [to_torch(x, dtype) for x in ins]
    got = [torch.zeros_like(src[0]) for _ in range(p)]
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    saved = {k: os.environ.get(k) for k in ("SIMCOMM_FAULT_SKIP_RANK", "SIMCOMM_TIMEOUT_NS")}
    try:
        os.environ["SIMCOMM_FAULT_SKIP_RANK"] = "1"
        os.environ["SIMCOMM_TIMEOUT_NS"] = "50000000"
        noalloc(L, src, got, n, dtype, op, status)
        torch.cuda.synchronize()
        assert int(status.item()) == SC.TIMEOUT
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    noalloc(L, src, got, n, dtype, op, status)
    torch.cuda.synchronize()
    assert int(status.item()) == SC.OK
    want = O.ring_allreduce(ins, dtype, op)
    for r in range(p):
        np.testing.assert_array_equal(bits(to_numpy(got[r], dtype)), bits(want[r]))


CHILD = textwrap.dedent("""
    import ctypes, sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import oracle as O
    from collective_communication_primitives_b200 import simcomm as SC
    from gpu_helpers import make_inputs, to_numpy, to_torch
    L = SC.load_library()
    p, n = 8, 300_001
    ins = make_inputs("normal", p, n, "bf16", "noalloc.child", sigma=1e-3)
    src = [to_torch(x, "bf16") for x in ins]
    got = [torch.zeros_like(src[0]) for _ in range(p)]
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    s = (ctypes.c_void_p * p)(*[t.data_ptr() for t in src])
    r = (ctypes.c_void_p * p)(*[t.data_ptr() for t in got])
    bufs = SC._Bufs(ctypes.cast(s, ctypes.POINTER(ctypes.c_void_p)), ctypes.cast(r, ctypes.POINTER(ctypes.c_void_p)))
    for call in range(2):
        rc = L.coll_allreduce_ring_noalloc(p, bufs, n, SC.DTYPES["bf16"], SC.OPS["avg"],
                                           ctypes.c_void_p(status.data_ptr()),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == SC.OK, L.sim_comm_last_error()
        torch.cuda.synchronize()
        assert int(status.item()) == SC.OK
        want = O.ring_allreduce(ins, "bf16", "avg")
        for q in range(p):
            assert np.array_equal(to_numpy(got[q], "bf16"), want[q]), (call, q)
    print("child ok")
""")


def test_noalloc_first_call_in_a_process_without_a_communicator():
    """The case the entry point exists for: a process whose first library call is this one, with no
    communicator ever created, so the scratch address is looked up by that call."""
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    env = {k: v for k, v in os.environ.items() if not k.startswith("SIMCOMM_")}
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "child ok" in res.stdout
