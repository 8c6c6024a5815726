"""The C-ABI library builds, loads and exports every entry point include/simcomm.h declares; the
host-side argument checks work without a GPU."""
import ctypes
import os
import re

import pytest

from collective_communication_primitives_b200 import build as B
from collective_communication_primitives_b200 import simcomm as SC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "simcomm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)) - {"defined"})


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ctypes.CDLL(B.LIB)


def test_header_declares_the_collectives():
    names = declared_functions()
    for want in ("sim_comm_create", "sim_comm_destroy", "coll_allreduce", "coll_reduce", "coll_broadcast",
                 "coll_reduce_scatter", "coll_allgather", "coll_alltoall", "coll_alltoallv",
                 "sim_comm_get_async_error", "sim_comm_abort", "sim_comm_reset"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    missing = [f for f in declared_functions() if not hasattr(lib, f)]
    assert not missing, missing


def test_binding_declares_every_symbol(lib):
    L = SC.load_library()
    for f in declared_functions():
        assert getattr(L, f).restype is not None or f in ("sim_comm_last_error",)


def test_status_strings(lib):
    L = SC.load_library()
    for code, name in SC.STATUS.items():
        assert L.coll_status_string(code).decode() == name


def test_null_communicator_is_rejected_without_a_gpu(lib):
    """Every entry point that takes a communicator refuses a NULL one before touching the device."""
    L = SC.load_library()
    bufs = SC._Bufs()
    assert L.coll_allreduce(None, bufs, 16, 1, 0, 0, None) == SC.INVALID_ARG
    assert L.coll_reduce(None, bufs, 16, 1, 0, 0, 0, None) == SC.INVALID_ARG
    assert L.coll_broadcast(None, bufs, 16, 1, 0, 0, None) == SC.INVALID_ARG
    assert L.coll_reduce_scatter(None, bufs, 16, 1, 0, 0, None) == SC.INVALID_ARG
    assert L.coll_allgather(None, bufs, 16, 1, 0, None) == SC.INVALID_ARG
    assert L.coll_alltoall(None, bufs, 16, 1, 0, None) == SC.INVALID_ARG
    assert L.coll_scatter(None, bufs, 16, 1, 0, 0, None) == SC.INVALID_ARG
    assert L.coll_gather(None, bufs, 16, 1, 0, 0, None) == SC.INVALID_ARG
    assert L.coll_alltoallv(None, bufs, None, None, None, 1, 0, None, None) == SC.INVALID_ARG
    assert L.coll_moe_dispatch(None, None, None, 4, 2, 8, 4, 2, None, 16, None, None, None, None) == SC.INVALID_ARG
    assert L.coll_moe_combine(None, None, 16, None, None, None, None, 4, 2, 8, 4, 2, None, None) == SC.INVALID_ARG
    v = ctypes.c_longlong()
    assert L.sim_comm_set_option(None, b"trace", 1) == SC.INVALID_ARG
    assert L.sim_comm_get_option(None, b"trace", ctypes.byref(v)) == SC.INVALID_ARG
    st = ctypes.c_int()
    assert L.sim_comm_get_async_error(None, ctypes.byref(st)) == SC.INVALID_ARG
    assert L.sim_comm_reset(None) == SC.INVALID_ARG
    n = ctypes.c_ulonglong()
    assert L.sim_comm_launch_count(None, ctypes.byref(n)) == SC.INVALID_ARG
    assert L.sim_comm_size(None) == -1
    assert L.sim_comm_destroy(None) == SC.OK
    assert L.sim_comm_abort(None) == SC.INVALID_ARG


def test_create_rejects_bad_rank_counts(lib):
    L = SC.load_library()
    assert not L.sim_comm_create(0)
    assert b"p must be" in L.sim_comm_last_error()
    assert not L.sim_comm_create(65)


def header_enum(prefix):
    text = open(os.path.join(ROOT, "include", "simcomm.h")).read()
    return {m.group(1): int(m.group(2)) for m in re.finditer(rf"\b{prefix}(\w+)\s*=\s*(\d+)", text)}


def test_binding_codes_match_the_header():
    algos = header_enum("COLL_ALGO_")
    names = {"direct": "DIRECT", "ring": "RING", "rd": "RD", "hd": "HD", "tree": "TREE", "dbtree": "DBTREE",
             "ll": "RING_LL", "rd_ll": "RD_LL", "tree_ll": "TREE_LL",
             "dbtree_ll": "DBTREE_LL"}
    assert set(names.values()) == set(algos)
    for key, hname in names.items():
        assert SC.ALGOS[key] == algos[hname], key
    dtypes = header_enum("COLL_")
    assert SC.DTYPES == {"int32": dtypes["INT32"], "fp32": dtypes["FP32"], "bf16": dtypes["BF16"]}
    assert SC.OPS == {"sum": dtypes["SUM"], "min": dtypes["MIN"], "max": dtypes["MAX"], "avg": dtypes["AVG"]}
    status = header_enum("COLL_ERR_")
    status["OK"] = header_enum("COLL_")["OK"]
    assert {v: "COLL_ERR_" + k if k != "OK" else "COLL_OK" for k, v in status.items()} == SC.STATUS


def test_trace_record_layout_matches_the_header(tmp_path):
    """The binding's TraceRecord has the offsets and size that a C compiler gives the header's
    sim_comm_trace_record_t."""
    import subprocess
    fields = [name for name, _ in SC.TraceRecord._fields_]
    src = tmp_path / "layout.c"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    body = "".join(f'    printf("%zu ", offsetof(sim_comm_trace_record_t, {f}));\n' for f in fields)
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"simcomm.h\"\nint main(void) {\n" + body +
                   '    printf("%zu\\n", sizeof(sim_comm_trace_record_t));\n    return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [getattr(SC.TraceRecord, f).offset for f in fields] + [ctypes.sizeof(SC.TraceRecord)]
    assert got == want


def test_trace_read_rejects_bad_arguments(lib):
    L = SC.load_library()
    count = ctypes.c_int(-1)
    assert L.sim_comm_trace_read(None, None, 0, ctypes.byref(count)) == SC.INVALID_ARG


def test_noalloc_entry_checks_its_arguments_without_a_gpu(lib):
    L = SC.load_library()
    bufs = SC._Bufs()
    assert L.coll_allreduce_ring_noalloc(1, bufs, 16, 1, 0, None, None) == SC.INVALID_ARG
    assert b"p must be" in L.sim_comm_last_error()
    assert L.coll_allreduce_ring_noalloc(65, bufs, 16, 1, 0, None, None) == SC.INVALID_ARG
    assert L.coll_allreduce_ring_noalloc(4, bufs, 16, 7, 0, None, None) == SC.INVALID_ARG
    assert L.coll_allreduce_ring_noalloc(4, bufs, 16, SC.DTYPES["int32"], SC.OPS["avg"], None, None) == SC.UNSUPPORTED


def test_noalloc_rejects_counts_whose_byte_sizes_would_wrap(lib):
    """n beyond 2^48 elements is refused before any size is formed: 2^62 fp32 elements would make
    n * 4 wrap to 0 bytes, which the pointer and scratch checks would then accept."""
    L = SC.load_library()
    p = 4
    fake = (ctypes.c_void_p * p)(*[0x7f0000000000 + 0x1000000 * r for r in range(p)])
    out = (ctypes.c_void_p * p)(*[0x7f8000000000 + 0x1000000 * r for r in range(p)])
    bufs = SC._Bufs(ctypes.cast(fake, ctypes.POINTER(ctypes.c_void_p)),
                    ctypes.cast(out, ctypes.POINTER(ctypes.c_void_p)))
    for n in (1 << 62, (1 << 48) + 1, (1 << 64) - 1):
        assert L.coll_allreduce_ring_noalloc(p, bufs, n, SC.DTYPES["fp32"], SC.OPS["sum"], None, None) == \
            SC.INVALID_ARG
        assert b"2^48" in L.sim_comm_last_error()
    nullbufs = SC._Bufs()  # refused on the size, before the NULL pointers are looked at
    assert L.coll_allreduce_ring_noalloc(p, nullbufs, 1 << 62, SC.DTYPES["fp32"], SC.OPS["sum"], None, None) == \
        SC.INVALID_ARG
    assert b"2^48" in L.sim_comm_last_error()


def test_rank_view_and_ipc_entries_check_their_arguments_without_a_gpu(lib):
    L = SC.load_library()
    assert not L.sim_comm_create_rank(4, 4)
    assert b"rank in [0, p)" in L.sim_comm_last_error()
    assert not L.sim_comm_create_rank(0, 0)
    assert not L.sim_comm_create_rank(4, -1)
    assert L.sim_comm_rank(None) == -2
    ptr = ctypes.c_void_p()
    h = SC.IpcHandle()
    assert L.sim_ipc_alloc(0, ctypes.byref(ptr), ctypes.byref(h)) == SC.INVALID_ARG
    assert L.sim_ipc_alloc(16, None, ctypes.byref(h)) == SC.INVALID_ARG
    assert L.sim_ipc_alloc((1 << 48) + 1, ctypes.byref(ptr), ctypes.byref(h)) == SC.INVALID_ARG
    assert L.sim_ipc_open(None, ctypes.byref(ptr)) == SC.INVALID_ARG
    assert L.sim_ipc_open(ctypes.byref(h), None) == SC.INVALID_ARG
    assert L.sim_ipc_free(None) == SC.OK and L.sim_ipc_close(None) == SC.OK
    assert ctypes.sizeof(SC.IpcHandle) == 64


def test_header_documents_every_option_the_library_accepts():
    """The option list in include/simcomm.h names exactly the keys the library takes (the key table
    in csrc/api.cu, which sim_comm_create also reads from the environment)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    header = open(os.path.join(root, "include", "simcomm.h")).read()
    start = header.index("/* Options (each also read from the environment")
    block = header[start:header.index("*/", start)]
    documented = set(re.findall(r'^ \*   "([a-z0-9_]+)"', block, flags=re.M))
    src = open(os.path.join(root, "collective_communication_primitives_b200", "csrc", "api.cu")).read()
    table = src[src.index("kOptionKeys[] = {"):]
    table = table[:table.index("};")]
    accepted = set(re.findall(r'"([a-z0-9_]+)"', table))
    assert documented == accepted, (sorted(documented - accepted), sorted(accepted - documented))
