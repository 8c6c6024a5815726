"""Python binding of the simulated-communicator library ``libsimcomm.so`` (C ABI: include/simcomm.h).

Argument marshalling only: tensors become device pointers and the current CUDA stream becomes the
stream handle; every step of every collective runs in the library's CUDA kernels. There is no
fallback: without the built library (``python -m collective_communication_primitives_b200.build``)
creating a communicator raises.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsimcomm.so")

STATUS = {0: "COLL_OK", 1: "COLL_ERR_INVALID_ARG", 2: "COLL_ERR_UNSUPPORTED", 3: "COLL_ERR_CUDA",
          4: "COLL_ERR_TIMEOUT", 5: "COLL_ERR_ABORTED", 6: "COLL_ERR_OVERFLOW", 7: "COLL_ERR_INTERNAL"}
OK, INVALID_ARG, UNSUPPORTED, CUDA, TIMEOUT, ABORTED, OVERFLOW, INTERNAL = range(8)
DTYPES = {"int32": 0, "fp32": 1, "bf16": 2}
OPS = {"sum": 0, "min": 1, "max": 2, "avg": 3}
ALGOS = {"direct": 0, "ring": 1, "rd": 2, "hd": 3, "tree": 4, "dbtree": 5, "ll": 6, "rd_ll": 7, "tree_ll": 8,
         "dbtree_ll": 9}

_lib = None


class SimCommError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class _Bufs(ctypes.Structure):
    _fields_ = [("send", ctypes.POINTER(ctypes.c_void_p)), ("recv", ctypes.POINTER(ctypes.c_void_p))]


class IpcHandle(ctypes.Structure):
    """sim_ipc_handle_t: 64 opaque bytes naming a shareable device buffer."""
    _fields_ = [("reserved", ctypes.c_ubyte * 64)]


class TraceRecord(ctypes.Structure):
    """sim_comm_trace_record_t: one traced call."""
    _fields_ = [("seq", ctypes.c_ulonglong), ("coll", ctypes.c_char_p), ("p", ctypes.c_int), ("dtype", ctypes.c_int),
                ("op", ctypes.c_int), ("root", ctypes.c_int), ("algo", ctypes.c_int), ("status", ctypes.c_int),
                ("n", ctypes.c_ulonglong), ("launches", ctypes.c_uint), ("device_ms", ctypes.c_float)]


def load_library(path=LIB_PATH):
    """Load libsimcomm.so and declare its signatures. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m collective_communication_primitives_b200.build`"
                           " (there is no fallback path)")
    L = ctypes.CDLL(path)
    vp, sz, i32, ll = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_longlong
    llp = ctypes.POINTER(ctypes.c_longlong)
    st = ctypes.c_int
    L.sim_comm_create.argtypes = [i32]
    L.sim_comm_create.restype = vp
    L.sim_comm_create_rank.argtypes = [i32, i32]
    L.sim_comm_create_rank.restype = vp
    L.sim_comm_rank.argtypes = [vp]
    L.sim_comm_rank.restype = i32
    L.sim_ipc_alloc.argtypes = [sz, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(IpcHandle)]
    L.sim_ipc_free.argtypes = [vp]
    L.sim_ipc_open.argtypes = [ctypes.POINTER(IpcHandle), ctypes.POINTER(ctypes.c_void_p)]
    L.sim_ipc_close.argtypes = [vp]
    for name in ("sim_ipc_alloc", "sim_ipc_free", "sim_ipc_open", "sim_ipc_close"):
        getattr(L, name).restype = ctypes.c_int
    L.sim_comm_destroy.argtypes = [vp]
    L.sim_comm_destroy.restype = st
    L.sim_comm_size.argtypes = [vp]
    L.sim_comm_size.restype = i32
    L.sim_comm_last_error.argtypes = []
    L.sim_comm_last_error.restype = ctypes.c_char_p
    L.coll_status_string.argtypes = [st]
    L.coll_status_string.restype = ctypes.c_char_p
    L.sim_comm_set_option.argtypes = [vp, ctypes.c_char_p, ll]
    L.sim_comm_set_option.restype = st
    L.sim_comm_get_option.argtypes = [vp, ctypes.c_char_p, llp]
    L.sim_comm_get_option.restype = st
    L.sim_comm_get_async_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    L.sim_comm_get_async_error.restype = st
    L.sim_comm_abort.argtypes = [vp]
    L.sim_comm_abort.restype = st
    L.sim_comm_reset.argtypes = [vp]
    L.sim_comm_reset.restype = st
    L.sim_comm_launch_count.argtypes = [vp, ctypes.POINTER(ctypes.c_ulonglong)]
    L.sim_comm_launch_count.restype = st
    L.sim_comm_trace_read.argtypes = [vp, ctypes.POINTER(TraceRecord), i32, ctypes.POINTER(ctypes.c_int)]
    L.sim_comm_trace_read.restype = st
    L.coll_allreduce.argtypes = [vp, _Bufs, sz, i32, i32, i32, vp]
    L.coll_reduce.argtypes = [vp, _Bufs, sz, i32, i32, i32, i32, vp]
    L.coll_broadcast.argtypes = [vp, _Bufs, sz, i32, i32, i32, vp]
    L.coll_reduce_scatter.argtypes = [vp, _Bufs, sz, i32, i32, i32, vp]
    L.coll_allgather.argtypes = [vp, _Bufs, sz, i32, i32, vp]
    L.coll_alltoall.argtypes = [vp, _Bufs, sz, i32, i32, vp]
    L.coll_alltoallv.argtypes = [vp, _Bufs, vp, llp, llp, i32, i32, vp, vp]
    L.coll_scatter.argtypes = [vp, _Bufs, sz, i32, i32, i32, vp]
    L.coll_gather.argtypes = [vp, _Bufs, sz, i32, i32, i32, vp]
    L.coll_allreduce_ring_noalloc.argtypes = [i32, _Bufs, sz, i32, i32, vp, vp]
    L.sim_hbm_probe.argtypes = [i32, vp, vp, sz, i32, vp]
    pp = ctypes.POINTER(ctypes.c_void_p)
    L.coll_moe_dispatch.argtypes = [vp, pp, pp, sz, i32, sz, i32, i32, pp, sz, pp, vp, vp, vp]
    L.coll_moe_combine.argtypes = [vp, pp, sz, pp, pp, pp, pp, sz, i32, sz, i32, i32, pp, vp]
    for name in ("coll_allreduce", "coll_reduce", "coll_broadcast", "coll_reduce_scatter", "coll_allgather",
                 "coll_alltoall", "coll_alltoallv", "coll_scatter", "coll_gather", "coll_allreduce_ring_noalloc",
                 "coll_moe_dispatch", "coll_moe_combine", "sim_hbm_probe"):
        getattr(L, name).restype = st
    _lib = L
    return L


def _ptr(x):
    """Device address of a tensor (or an int address, or None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _dtype_of(t):
    import torch
    m = {torch.int32: "int32", torch.float32: "fp32", torch.bfloat16: "bf16"}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


class SimComm:
    """A communicator of p logical ranks on the current CUDA device (or, with `rank`, the rank view
    that the process of that rank holds when every rank is its own process)."""

    def __init__(self, p, rank=None):
        self._L = load_library()
        h = self._L.sim_comm_create(int(p)) if rank is None else self._L.sim_comm_create_rank(int(p), int(rank))
        if not h:
            raise SimCommError(CUDA if rank is None else INVALID_ARG, self._L.sim_comm_last_error().decode())
        self._h = ctypes.c_void_p(h)
        self.p = int(p)
        self.rank = None if rank is None else int(rank)

    # -- lifecycle ---------------------------------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            self._L.sim_comm_destroy(self._h)
            self._h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, status):
        if status != OK:
            raise SimCommError(status, self._L.sim_comm_last_error().decode())

    def set_option(self, key, value):
        self._check(self._L.sim_comm_set_option(self._h, key.encode(), int(value)))

    def get_option(self, key):
        v = ctypes.c_longlong()
        self._check(self._L.sim_comm_get_option(self._h, key.encode(), ctypes.byref(v)))
        return v.value

    def async_error(self):
        s = ctypes.c_int()
        self._check(self._L.sim_comm_get_async_error(self._h, ctypes.byref(s)))
        return s.value

    def abort(self):
        self._check(self._L.sim_comm_abort(self._h))

    def reset(self):
        self._check(self._L.sim_comm_reset(self._h))

    def launch_count(self):
        v = ctypes.c_ulonglong()
        self._check(self._L.sim_comm_launch_count(self._h, ctypes.byref(v)))
        return v.value

    def trace_read(self, cap=4096):
        """The traced calls not read yet (option "trace" = 1), oldest first, as dicts with the fields of
        sim_comm_trace_record_t (coll decoded to str). Waits for their events."""
        buf = (TraceRecord * cap)()
        got = ctypes.c_int()
        self._check(self._L.sim_comm_trace_read(self._h, buf, cap, ctypes.byref(got)))
        out = []
        for r in buf[:got.value]:
            d = {name: getattr(r, name) for name, _ in TraceRecord._fields_}
            d["coll"] = d["coll"].decode()
            out.append(d)
        return out

    # -- marshalling -------------------------------------------------------------------------------
    def _bufs(self, sends, recvs):
        p = self.p
        s = (ctypes.c_void_p * p)(*[_ptr(x) for x in sends])
        r = (ctypes.c_void_p * p)(*[_ptr(x) for x in recvs])
        self._keep = (s, r)
        return _Bufs(ctypes.cast(s, ctypes.POINTER(ctypes.c_void_p)), ctypes.cast(r, ctypes.POINTER(ctypes.c_void_p)))

    @staticmethod
    def _resolve(dtype, tensors):
        if dtype is not None:
            return DTYPES[dtype]
        for t in tensors:
            if t is not None and not isinstance(t, int):
                return DTYPES[_dtype_of(t)]
        raise ValueError("dtype is needed when only raw pointers are given")

    # -- collectives (n follows include/simcomm.h: the per-rank FULL buffer) -----------------------
    def allreduce(self, sends, recvs, op="sum", algo="direct", n=None, dtype=None, stream=None):
        n = sends[0].numel() if n is None else n
        self._check(self._L.coll_allreduce(self._h, self._bufs(sends, recvs), n, self._resolve(dtype, list(sends) + list(recvs)),
                                           OPS[op], ALGOS[algo], _stream(stream)))

    def reduce(self, sends, recvs, root, op="sum", algo="direct", n=None, dtype=None, stream=None):
        n = sends[0].numel() if n is None else n
        self._check(self._L.coll_reduce(self._h, self._bufs(sends, recvs), n, self._resolve(dtype, list(sends) + list(recvs)), OPS[op],
                                        int(root), ALGOS[algo], _stream(stream)))

    def broadcast(self, sends, recvs, root, algo="direct", n=None, dtype=None, stream=None):
        n = recvs[0].numel() if n is None else n
        self._check(self._L.coll_broadcast(self._h, self._bufs(sends, recvs), n, self._resolve(dtype, list(sends) + list(recvs)),
                                           int(root), ALGOS[algo], _stream(stream)))

    def reduce_scatter(self, sends, recvs, op="sum", algo="direct", n=None, dtype=None, stream=None):
        n = sends[0].numel() if n is None else n
        self._check(self._L.coll_reduce_scatter(self._h, self._bufs(sends, recvs), n, self._resolve(dtype, list(sends) + list(recvs)),
                                                OPS[op], ALGOS[algo], _stream(stream)))

    def allgather(self, sends, recvs, algo="direct", n=None, dtype=None, stream=None):
        n = recvs[0].numel() if n is None else n
        self._check(self._L.coll_allgather(self._h, self._bufs(sends, recvs), n, self._resolve(dtype, list(sends) + list(recvs)),
                                           ALGOS[algo], _stream(stream)))

    def alltoall(self, sends, recvs, algo="direct", n=None, dtype=None, stream=None):
        n = sends[0].numel() if n is None else n
        self._check(self._L.coll_alltoall(self._h, self._bufs(sends, recvs), n, self._resolve(dtype, list(sends) + list(recvs)),
                                          ALGOS[algo], _stream(stream)))

    def scatter(self, sends, recvs, root, algo="direct", n=None, dtype=None, stream=None):
        """n: the root's full buffer (p blocks); only sends[root] is read."""
        n = sends[root].numel() if n is None else n
        self._check(self._L.coll_scatter(self._h, self._bufs(sends, recvs), n,
                                         self._resolve(dtype, list(sends) + list(recvs)), int(root), ALGOS[algo],
                                         _stream(stream)))

    def gather(self, sends, recvs, root, algo="direct", n=None, dtype=None, stream=None):
        """n: the root's full buffer (p blocks); only recvs[root] is written."""
        n = recvs[root].numel() if n is None else n
        self._check(self._L.coll_gather(self._h, self._bufs(sends, recvs), n,
                                        self._resolve(dtype, list(sends) + list(recvs)), int(root), ALGOS[algo],
                                        _stream(stream)))

    def alltoallv(self, sends, recvs, counts, send_cap=None, recv_cap=None, algo="direct", recv_counts=None,
                  dtype=None, stream=None):
        """counts: device int64 [p][p] tensor (c[i][j] elements from i to j). Capacities default to the
        buffers' sizes."""
        p = self.p
        send_cap = [sends[i].numel() for i in range(p)] if send_cap is None else send_cap
        recv_cap = [recvs[j].numel() for j in range(p)] if recv_cap is None else recv_cap
        sc = (ctypes.c_longlong * p)(*[int(x) for x in send_cap])
        rc = (ctypes.c_longlong * p)(*[int(x) for x in recv_cap])
        self._check(self._L.coll_alltoallv(self._h, self._bufs(sends, recvs), ctypes.c_void_p(_ptr(counts)), sc, rc,
                                           self._resolve(dtype, list(sends) + list(recvs)), ALGOS[algo], _stream(stream),
                                           ctypes.c_void_p(_ptr(recv_counts)) if recv_counts is not None else None))

    # -- MoE dispatch / combine ----------------------------------------------------------------------
    def _parr(self, tensors):
        """HOST array of p device pointers (None when tensors is None)."""
        if tensors is None:
            return None
        a = (ctypes.c_void_p * self.p)(*[_ptr(t) for t in tensors])
        self._keep_moe = getattr(self, "_keep_moe", [])[-16:] + [a]
        return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))

    def moe_dispatch(self, x, topk_idx, experts, recv, route_pos=None, expert_counts=None, recv_counts=None,
                     dtype=None, stream=None):
        """x[i]: [T][H] token rows; topk_idx[i]: [T][k] int32 expert ids; recv[j]: [cap][H]. Optional
        outputs: route_pos[i] [T][k] int32, expert_counts [p][E] int64, recv_counts [p] int64."""
        T, k = topk_idx[0].shape
        H = x[0].shape[1] if x[0].dim() == 2 else x[0].numel() // max(T, 1)
        cap = recv[0].shape[0]
        self._check(self._L.coll_moe_dispatch(
            self._h, self._parr(x), self._parr(topk_idx), T, k, H, int(experts),
            self._resolve(dtype, list(x) + list(recv)), self._parr(recv), cap, self._parr(route_pos),
            ctypes.c_void_p(_ptr(expert_counts)) if expert_counts is not None else None,
            ctypes.c_void_p(_ptr(recv_counts)) if recv_counts is not None else None, _stream(stream)))

    def moe_combine(self, y, topk_idx, route_pos, topk_weight, experts, out, residual=None, dtype=None,
                    stream=None):
        """out[i][t] = residual[i][t] + Σ_s w[i][t][s] * y[owner][route_pos[i][t][s]] (fp32, slot order)."""
        T, k = topk_idx[0].shape
        H = out[0].shape[1]
        self._check(self._L.coll_moe_combine(
            self._h, self._parr(y), y[0].shape[0], self._parr(topk_idx), self._parr(route_pos),
            self._parr(topk_weight), self._parr(residual), T, k, H, int(experts),
            self._resolve(dtype, list(y) + list(out)), self._parr(out), _stream(stream)))


def allreduce_ring_noalloc(sends, recvs, op="sum", n=None, dtype=None, status=None, stream=None):
    """Ring AllReduce on the library's static scratch: no communicator, no allocation (for callers
    that cannot allocate device memory; see include/simcomm.h). `status` is an optional device int32
    tensor that receives the call's asynchronous status."""
    L = load_library()
    p = len(sends)
    n = sends[0].numel() if n is None else n
    s = (ctypes.c_void_p * p)(*[_ptr(x) for x in sends])
    r = (ctypes.c_void_p * p)(*[_ptr(x) for x in recvs])
    bufs = _Bufs(ctypes.cast(s, ctypes.POINTER(ctypes.c_void_p)), ctypes.cast(r, ctypes.POINTER(ctypes.c_void_p)))
    dt = SimComm._resolve(dtype, list(sends) + list(recvs))
    rc = L.coll_allreduce_ring_noalloc(p, bufs, n, dt, OPS[op], ctypes.c_void_p(_ptr(status)) if status is not None
                                       else None, _stream(stream))
    if rc != OK:
        raise SimCommError(rc, L.sim_comm_last_error().decode())


PROBES = {"load": 0, "store": 1, "copy": 2, "bulk_store": 3, "bulk_fanout": 4}


def hbm_probe(kind, dst, src, nbytes, ctas_per_sm, stream=None):
    """One HBM access-pattern probe (sim_hbm_probe): `kind` in PROBES; dst/src device tensors (or None
    where the kind does not use them), nbytes a multiple of 16 KiB (bulk_fanout: of 32 KiB, and dst
    holds 8 * nbytes)."""
    L = load_library()
    rc = L.sim_hbm_probe(PROBES[kind], ctypes.c_void_p(_ptr(dst)) if dst is not None else None,
                         ctypes.c_void_p(_ptr(src)) if src is not None else None, nbytes, ctas_per_sm,
                         _stream(stream))
    if rc != OK:
        raise SimCommError(rc, L.sim_comm_last_error().decode())
