"""The per-call trace (option "trace", sim_comm_trace_read) and the options read from the
environment at create time."""
import os

import pytest
import torch

from collective_communication_primitives_b200 import simcomm as SC

pytestmark = pytest.mark.gpu


def test_trace_records_every_call_in_order():
    p, n = 4, 1 << 16
    c = SC.SimComm(p)
    try:
        assert c.get_option("trace") == 0
        x = [torch.ones(n, device="cuda") for _ in range(p)]
        y = [torch.empty(n, device="cuda") for _ in range(p)]
        c.allreduce(x, y)  # not traced
        c.set_option("trace", 1)
        c.allreduce(x, y, op="max", algo="ring")
        c.broadcast(x, y, 2)
        with pytest.raises(SC.SimCommError):
            c.reduce(x, y, root=p)  # refused before any launch
        c.allgather([t[: n // p] for t in x], y, algo="ring")
        c.set_option("trace", 0)
        c.allreduce(x, y)  # not traced
        recs = c.trace_read()
        assert [r["coll"] for r in recs] == ["allreduce", "broadcast", "reduce", "allgather"]
        assert [r["seq"] for r in recs] == [0, 1, 2, 3]
        ar, bc, bad, ag = recs
        assert (ar["p"], ar["n"], ar["dtype"], ar["op"], ar["root"], ar["algo"]) == (p, n, 1, 2, -1, SC.ALGOS["ring"])
        assert (bc["root"], bc["algo"], bc["op"]) == (2, SC.ALGOS["direct"], -1)
        assert bad["status"] == SC.INVALID_ARG and bad["launches"] == 0 and bad["device_ms"] == -1.0
        for r in (ar, bc, ag):
            assert r["status"] == SC.OK and r["launches"] >= 1 and r["device_ms"] > 0
        assert c.trace_read() == []  # read once
    finally:
        c.close()


def test_trace_keeps_the_last_4096_calls():
    p, n = 2, 256
    c = SC.SimComm(p)
    try:
        c.set_option("trace", 1)
        x = [torch.ones(n, device="cuda") for _ in range(p)]
        y = [torch.empty(n, device="cuda") for _ in range(p)]
        for _ in range(4096 + 10):
            c.allreduce(x, y)
        recs = c.trace_read(cap=5000)
        assert len(recs) == 4096
        assert [r["seq"] for r in recs] == list(range(10, 4106))
        assert all(r["device_ms"] > 0 for r in recs)
    finally:
        c.close()


def test_options_from_the_environment():
    keys = {"SIMCOMM_TRACE": "1", "SIMCOMM_COPY_ORDER": "0", "SIMCOMM_RING_TASK_BYTES": "65536",
            "SIMCOMM_CHUNK_BYTES": "12345"}  # the last one is rejected (not a multiple of 256): default stays
    old = {k: os.environ.get(k) for k in keys}
    os.environ.update(keys)
    try:
        c = SC.SimComm(2)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    try:
        assert c.get_option("trace") == 1
        assert c.get_option("copy_order") == 0
        assert c.get_option("ring_task_bytes") == 65536
        assert c.get_option("chunk_bytes") == 1 << 20
    finally:
        c.close()
