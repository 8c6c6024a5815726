"""CPU oracle for the simulated-communicator collectives -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import this
package. The product (the CUDA library and its Python binding) never imports, links or calls it.

This module only marshals numpy arrays into ``liboracle.so`` (built from ``oracle.cpp``), where the
definitions live. bf16 arrays are passed as ``numpy.uint16`` bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

DTYPE_CODES = {"int32": 0, "fp32": 1, "bf16": 2}
OP_CODES = {"sum": 0, "min": 1, "max": 2, "avg": 3}
ACC_CODES = {"exact": 0, "rankfold": 1, "slotfold": 1}
NP_DTYPES = {"int32": np.int32, "fp32": np.float32, "bf16": np.uint16}


def lib():
    global _LIB
    if _LIB is None:
        # ORACLE_LIB points at another build of oracle.cpp (the mutation tests plant mistakes in a
        # copy and check that the pins catch them).
        path = os.environ.get("ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        pp = ctypes.POINTER(ctypes.c_void_p)
        i64p = ctypes.POINTER(ctypes.c_int64)
        sigs = {
            "oracle_allreduce": [i32, pp, pp, sz, i32, i32, i32],
            "oracle_reduce": [i32, pp, vp, sz, i32, i32, i32, i32],
            "oracle_broadcast": [i32, vp, pp, sz, i32, i32],
            "oracle_reduce_scatter": [i32, pp, pp, sz, i32, i32, i32],
            "oracle_allgather": [i32, pp, pp, sz, i32],
            "oracle_alltoall": [i32, pp, pp, sz, i32],
            "oracle_alltoallv": [i32, pp, pp, i64p, i32, i64p],
            "oracle_ring_allreduce": [i32, pp, pp, sz, i32, i32],
            "oracle_ring_reduce_scatter": [i32, pp, pp, sz, i32, i32],
            "oracle_ring_allgather": [i32, pp, pp, sz, i32],
            "oracle_ring_reduce": [i32, pp, vp, sz, i32, i32, i32],
            "oracle_ring_broadcast": [i32, vp, pp, sz, i32, i32],
            "oracle_ring_alltoall": [i32, pp, pp, sz, i32],
            "oracle_scatter": [i32, vp, pp, sz, i32, i32],
            "oracle_gather": [i32, pp, vp, sz, i32, i32],
            "oracle_rd_allreduce": [i32, pp, pp, sz, i32, i32],
            "oracle_hd_allreduce": [i32, pp, pp, sz, i32, i32],
            "oracle_tree_allreduce": [i32, pp, pp, sz, i32, i32, i32],
            "oracle_moe_dispatch": [i32, pp, pp, sz, i32, sz, i32, i32, sz, pp, i64p, pp, i64p],
            "oracle_moe_combine": [i32, pp, pp, pp, pp, sz, i32, sz, i32, i32, pp, i32],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.oracle_float_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_float_to_bf16.restype = ctypes.c_uint16
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_float.restype = ctypes.c_float
        L.oracle_ring_segment.argtypes = [sz, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.oracle_ring_segment.restype = None
        _LIB = L
    return _LIB


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: arguments outside the oracle's definitions")


def _arr(x, dtype):
    a = np.ascontiguousarray(x)
    if a.dtype != NP_DTYPES[dtype]:
        raise TypeError(f"expected {NP_DTYPES[dtype]} for {dtype}, got {a.dtype}")
    return a


def _ptrs(arrays):
    return (ctypes.c_void_p * len(arrays))(*[a.ctypes.data for a in arrays])


def _outs(p, count, dtype):
    return [np.zeros(count, dtype=NP_DTYPES[dtype]) for _ in range(p)]


def allreduce(inputs, dtype, op, acc="exact"):
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    outs = _outs(len(ins), n, dtype)
    _check(lib().oracle_allreduce(len(ins), _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op],
                                  ACC_CODES[acc]), "allreduce")
    return outs


def reduce(inputs, dtype, op, root, acc="exact", out=None):
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    res = np.zeros(n, dtype=NP_DTYPES[dtype]) if out is None else out
    _check(lib().oracle_reduce(len(ins), _ptrs(ins), res.ctypes.data, n, DTYPE_CODES[dtype], OP_CODES[op], root,
                               ACC_CODES[acc]), "reduce")
    return res


def broadcast(root_input, p, dtype, root):
    x = _arr(root_input, dtype)
    outs = _outs(p, x.size, dtype)
    _check(lib().oracle_broadcast(p, x.ctypes.data, _ptrs(outs), x.size, DTYPE_CODES[dtype], root), "broadcast")
    return outs


def reduce_scatter(inputs, dtype, op, acc="exact"):
    ins = [_arr(x, dtype) for x in inputs]
    p, n = len(ins), ins[0].size
    outs = _outs(p, n // p, dtype)
    _check(lib().oracle_reduce_scatter(p, _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op],
                                       ACC_CODES[acc]), "reduce_scatter")
    return outs


def allgather(shards, dtype):
    ins = [_arr(x, dtype) for x in shards]
    p = len(ins)
    n = p * ins[0].size
    outs = _outs(p, n, dtype)
    _check(lib().oracle_allgather(p, _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype]), "allgather")
    return outs


def alltoall(inputs, dtype):
    ins = [_arr(x, dtype) for x in inputs]
    p, n = len(ins), ins[0].size
    outs = _outs(p, n, dtype)
    _check(lib().oracle_alltoall(p, _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype]), "alltoall")
    return outs


def alltoallv(inputs, counts, dtype):
    """counts: [p][p] int64, c[i][j] elements from source i to destination j. Returns
    (outputs sized Σ_i c_ij per destination j, recv_counts)."""
    ins = [_arr(x, dtype) for x in inputs]
    p = len(ins)
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.int64).reshape(p, p))
    recv = c.sum(axis=0)
    outs = [np.zeros(int(recv[j]), dtype=NP_DTYPES[dtype]) for j in range(p)]
    rc = np.zeros(p, dtype=np.int64)
    i64p = ctypes.POINTER(ctypes.c_int64)
    _check(lib().oracle_alltoallv(p, _ptrs(ins), _ptrs(outs), c.ctypes.data_as(i64p), DTYPE_CODES[dtype],
                                  rc.ctypes.data_as(i64p)), "alltoallv")
    return outs, rc


def scatter(root_input, p, dtype, root):
    """Scatter: block r of the root's [p·m] buffer goes to rank r."""
    x = _arr(root_input, dtype)
    outs = _outs(p, x.size // p, dtype)
    _check(lib().oracle_scatter(p, x.ctypes.data, _ptrs(outs), x.size, DTYPE_CODES[dtype], root), "scatter")
    return outs


def gather(inputs, dtype, root):
    """Gather: rank r's [m] block lands at block r of the root's [p·m] buffer."""
    ins = [_arr(x, dtype) for x in inputs]
    p = len(ins)
    n = p * ins[0].size
    res = np.zeros(n, dtype=NP_DTYPES[dtype])
    _check(lib().oracle_gather(p, _ptrs(ins), res.ctypes.data, n, DTYPE_CODES[dtype], root), "gather")
    return res


def ring_allreduce(inputs, dtype, op):
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    outs = _outs(len(ins), n, dtype)
    _check(lib().oracle_ring_allreduce(len(ins), _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op]),
           "ring_allreduce")
    return outs


def ring_reduce_scatter(inputs, dtype, op):
    ins = [_arr(x, dtype) for x in inputs]
    p, n = len(ins), ins[0].size
    outs = _outs(p, n // p, dtype)
    _check(lib().oracle_ring_reduce_scatter(p, _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op]),
           "ring_reduce_scatter")
    return outs


def ring_allgather(shards, dtype):
    ins = [_arr(x, dtype) for x in shards]
    p = len(ins)
    n = p * ins[0].size
    outs = _outs(p, n, dtype)
    _check(lib().oracle_ring_allgather(p, _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype]), "ring_allgather")
    return outs


def ring_reduce(inputs, dtype, op, root):
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    res = np.zeros(n, dtype=NP_DTYPES[dtype])
    _check(lib().oracle_ring_reduce(len(ins), _ptrs(ins), res.ctypes.data, n, DTYPE_CODES[dtype], OP_CODES[op],
                                    root), "ring_reduce")
    return res


def ring_broadcast(root_input, p, dtype, root):
    x = _arr(root_input, dtype)
    outs = _outs(p, x.size, dtype)
    _check(lib().oracle_ring_broadcast(p, x.ctypes.data, _ptrs(outs), x.size, DTYPE_CODES[dtype], root),
           "ring_broadcast")
    return outs


def ring_alltoall(inputs, dtype):
    ins = [_arr(x, dtype) for x in inputs]
    p, n = len(ins), ins[0].size
    outs = _outs(p, n, dtype)
    _check(lib().oracle_ring_alltoall(p, _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype]), "ring_alltoall")
    return outs


def rd_allreduce(inputs, dtype, op):
    """Recursive-doubling AllReduce (p a power of two)."""
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    outs = _outs(len(ins), n, dtype)
    _check(lib().oracle_rd_allreduce(len(ins), _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op]),
           "rd_allreduce")
    return outs


def hd_allreduce(inputs, dtype, op):
    """Recursive halving-doubling AllReduce (p a power of two)."""
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    outs = _outs(len(ins), n, dtype)
    _check(lib().oracle_hd_allreduce(len(ins), _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op]),
           "hd_allreduce")
    return outs


def tree_allreduce(inputs, dtype, op, double_tree=False):
    """Tree AllReduce: reduce up a heap-numbered binary tree, broadcast down; the double tree runs
    the second half of the elements on the mirrored tree."""
    ins = [_arr(x, dtype) for x in inputs]
    n = ins[0].size
    outs = _outs(len(ins), n, dtype)
    _check(lib().oracle_tree_allreduce(len(ins), _ptrs(ins), _ptrs(outs), n, DTYPE_CODES[dtype], OP_CODES[op],
                                       1 if double_tree else 0), "tree_allreduce")
    return outs


def moe_dispatch(x, idx, experts, cap_rows, dtype):
    """MoE dispatch: count -> exchange counts -> prefix sums -> pack/permute -> Alltoallv.

    x: p arrays [T][H] (token rows of each source rank); idx: p int32 arrays [T][k] of expert ids.
    Returns dict(recv=[p arrays [cap_rows][H]], expert_counts=[p][E], pos=[p arrays [T][k]] (row of
    each assignment in its owner's receive buffer), recv_counts=[p]); raises OverflowError when a
    destination would receive more than cap_rows rows."""
    xs = [_arr(a, dtype) for a in x]
    ids = [np.ascontiguousarray(a, dtype=np.int32) for a in idx]
    p = len(xs)
    T, k = ids[0].shape
    H = xs[0].shape[1] if xs[0].ndim == 2 else (xs[0].size // T if T else 0)
    recv = [np.zeros((cap_rows, H), dtype=NP_DTYPES[dtype]) for _ in range(p)]
    pos = [np.full((T, k), -1, dtype=np.int32) for _ in range(p)]
    ec = np.zeros((p, experts), dtype=np.int64)
    rc = np.zeros(p, dtype=np.int64)
    i64p = ctypes.POINTER(ctypes.c_int64)
    status = lib().oracle_moe_dispatch(p, _ptrs(xs), _ptrs(ids), T, k, H, experts, DTYPE_CODES[dtype], cap_rows,
                                       _ptrs(recv), ec.ctypes.data_as(i64p), _ptrs(pos), rc.ctypes.data_as(i64p))
    if status == 1:
        raise OverflowError("a destination would receive more rows than its capacity")
    _check(status, "moe_dispatch")
    return {"recv": recv, "expert_counts": ec, "pos": pos, "recv_counts": rc}


def moe_combine(y, idx, weights, dtype, experts, residual=None, acc="exact"):
    """MoE combine: reverse Alltoallv -> unpermute -> weighted sum (+ residual).

    y: p arrays [rows][H] of expert outputs in the dispatch receive layout; idx: the router's expert
    ids [T][k]; weights: fp32 [T][k]; residual: None or p arrays [T][H]. acc "exact" (double,
    rounded once) or "slotfold" (fp32 left fold in slot order). Returns p arrays [T][H]."""
    ys = [_arr(a, dtype) for a in y]
    ids = [np.ascontiguousarray(a, dtype=np.int32) for a in idx]
    ws = [np.ascontiguousarray(a, dtype=np.float32) for a in weights]
    p = len(ys)
    T, k = ids[0].shape
    H = ys[0].shape[1]
    res = None if residual is None else [_arr(a, dtype) for a in residual]
    outs = [np.zeros((T, H), dtype=NP_DTYPES[dtype]) for _ in range(p)]
    _check(lib().oracle_moe_combine(p, _ptrs(ys), _ptrs(ids), _ptrs(ws), None if res is None else _ptrs(res), T, k, H,
                                    experts, DTYPE_CODES[dtype], _ptrs(outs), ACC_CODES[acc]), "moe_combine")
    return outs


def float_to_bf16(x):
    L = lib()
    a = np.asarray(x, dtype=np.float32).ravel()
    return np.array([L.oracle_float_to_bf16(float(v)) for v in a], dtype=np.uint16)


def double_to_bf16(x):
    L = lib()
    a = np.asarray(x, dtype=np.float64).ravel()
    return np.array([L.oracle_double_to_bf16(float(v)) for v in a], dtype=np.uint16)


def bf16_to_float(h):
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def ring_segment(n, p, k):
    b, e = ctypes.c_size_t(), ctypes.c_size_t()
    lib().oracle_ring_segment(n, p, k, ctypes.byref(b), ctypes.byref(e))
    return b.value, e.value
