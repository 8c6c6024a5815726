"""Rank views: one rank of a communicator whose ranks are separate processes (include/simcomm.h,
sim_comm_create_rank and sim_ipc_*), after "集合通信：原语、算法、NCCL 实现与拓扑映射" §3.1-§3.3: the
ranks exchange buffer handles once over a host channel, then each rank's collective reads the peers'
buffers directly.

Argument marshalling and host plumbing only: buffers come from the library (sim_ipc_alloc), their
handles travel through torch.distributed (any backend; gloo on the CPU is enough), and every step of
a collective runs in the library's kernels. The library does not order the ranks' calls, so each
collective here is bracketed by the same host synchronisation on every rank: the caller's stream is
synchronised and the ranks meet at a barrier before the call (every input is complete) and after it
(no rank modifies its input while a peer may still read it). A rank that never arrives makes the
others' barrier fail with the process group's timeout, which is raised as COLL_ERR_TIMEOUT.
"""
import ctypes

from . import simcomm as SC

TORCH_OF = {"int32": "int32", "fp32": "float32", "bf16": "bfloat16"}
BYTES = {"int32": 4, "fp32": 4, "bf16": 2}


class _CudaArray:
    """A raw device range seen by torch through __cuda_array_interface__ (no copy, no ownership)."""

    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False), "version": 3,
                                         "strides": None}


class SharedBuffer:
    """Device memory another process can map (sim_ipc_alloc); freed by close() or at exit."""

    def __init__(self, nbytes):
        L = SC.load_library()
        self._L = L
        self.nbytes = int(nbytes)
        ptr = ctypes.c_void_p()
        self._handle = SC.IpcHandle()
        rc = L.sim_ipc_alloc(self.nbytes, ctypes.byref(ptr), ctypes.byref(self._handle))
        if rc != SC.OK:
            raise SC.SimCommError(rc, L.sim_comm_last_error().decode())
        self.ptr = int(ptr.value)

    @property
    def handle(self):
        return bytes(self._handle.reserved)

    def view(self, dtype, numel=None, offset=0):
        """A torch tensor over this buffer: `numel` elements of `dtype` ("int32", "fp32", "bf16") from
        element `offset` on."""
        import torch
        d = BYTES[dtype]
        numel = (self.nbytes - offset * d) // d if numel is None else int(numel)
        if offset < 0 or (offset + numel) * d > self.nbytes:
            raise ValueError("view outside the buffer")
        raw = torch.as_tensor(_CudaArray(self.ptr + offset * d, numel * d), device="cuda")
        return raw.view(getattr(torch, TORCH_OF[dtype]))

    def close(self):
        if self.ptr:
            self._L.sim_ipc_free(ctypes.c_void_p(self.ptr))
            self.ptr = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def exchange(obj, group=None):
    """Every rank's `obj`, in rank order (torch.distributed all_gather_object)."""
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, obj, group=group)
    return out


def open_handles(handles, my_rank, my_ptr, opener):
    """Rank-ordered device pointers of one registered buffer: this rank's own pointer, and every other
    rank's buffer mapped through `opener(handle) -> pointer`."""
    return [my_ptr if q == my_rank else opener(h) for q, h in enumerate(handles)]


class RankComm(SC.SimComm):
    """The rank view of the calling process (rank = torch.distributed rank, p = world size)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.group = group
        super().__init__(dist.get_world_size(group), rank=dist.get_rank(group))
        self._opened = []

    def _open(self, handle):
        h = SC.IpcHandle()
        ctypes.memmove(h.reserved, handle, 64)
        ptr = ctypes.c_void_p()
        self._check(self._L.sim_ipc_open(ctypes.byref(h), ctypes.byref(ptr)))
        self._opened.append(int(ptr.value))
        return int(ptr.value)

    def register(self, buf):
        """Every rank's buffer of this registration, rank-ordered: this rank's own pointer, the peers'
        mapped here. Collective: every rank calls it with its own buffer."""
        return open_handles(exchange(buf.handle, self.group), self.rank, buf.ptr, self._open)

    def sync(self):
        """Stream synchronised, then a barrier of all ranks; a rank that does not arrive within the
        process group's timeout raises COLL_ERR_TIMEOUT."""
        import torch
        import torch.distributed as dist
        torch.cuda.current_stream().synchronize()
        try:
            dist.barrier(group=self.group)
        except Exception as e:  # the group's timeout or a peer that left
            raise SC.SimCommError(SC.TIMEOUT, f"rank barrier failed: {e}") from e

    def _outs(self, recv):
        r = [None] * self.p
        r[self.rank] = recv
        return r

    def _call(self, fn, *args, **kw):
        """Every rank meets both barriers even when the library refuses the call (then the refusal is
        raised after the second one), so the ranks stay in step."""
        self.sync()
        try:
            fn(*args, **kw)
        finally:
            self.sync()

    # every rank passes the registered input pointers of all ranks and its own output pointer
    def allreduce(self, sends, recv, n, dtype, op="sum", algo="direct"):
        self._call(super().allreduce, sends, self._outs(recv), op=op, algo=algo, n=n, dtype=dtype)

    def reduce(self, sends, recv, root, n, dtype, op="sum", algo="direct"):
        self._call(super().reduce, sends, self._outs(recv), root, op=op, algo=algo, n=n, dtype=dtype)

    def broadcast(self, sends, recv, root, n, dtype, algo="direct"):
        self._call(super().broadcast, sends, self._outs(recv), root, algo=algo, n=n, dtype=dtype)

    def reduce_scatter(self, sends, recv, n, dtype, op="sum", algo="direct"):
        self._call(super().reduce_scatter, sends, self._outs(recv), op=op, algo=algo, n=n, dtype=dtype)

    def allgather(self, sends, recv, n, dtype, algo="direct"):
        self._call(super().allgather, sends, self._outs(recv), algo=algo, n=n, dtype=dtype)

    def alltoall(self, sends, recv, n, dtype, algo="direct"):
        self._call(super().alltoall, sends, self._outs(recv), algo=algo, n=n, dtype=dtype)

    def scatter(self, sends, recv, root, n, dtype, algo="direct"):
        self._call(super().scatter, sends, self._outs(recv), root, algo=algo, n=n, dtype=dtype)

    def gather(self, sends, recv, root, n, dtype, algo="direct"):
        self._call(super().gather, sends, self._outs(recv), root, algo=algo, n=n, dtype=dtype)

    def alltoallv(self, sends, recv, counts, send_cap, recv_cap, dtype, algo="direct", recv_counts=None):
        """counts: this process's device copy of the whole int64 [p][p] count matrix (the same on every
        rank); send_cap / recv_cap: every rank's capacities, in elements."""
        self._call(super().alltoallv, sends, self._outs(recv), counts, send_cap=send_cap, recv_cap=recv_cap,
                   algo=algo, recv_counts=recv_counts, dtype=dtype)

    def moe_dispatch(self, xs, topk_idx, experts, recv, tokens, topk, hidden, dtype, recv_cap, route_pos=None,
                     expert_counts=None, recv_counts=None):
        """xs, topk_idx: every rank's registered token rows and expert ids (pointers); recv: this rank's
        receive buffer [recv_cap][hidden], route_pos: this rank's [tokens][topk] int32 routing map or
        None; expert_counts / recv_counts: this process's int64 [p][E] / [p] outputs or None."""
        L = self._L

        def go():
            self._check(L.coll_moe_dispatch(
                self._h, self._parr(xs), self._parr(topk_idx), tokens, topk, hidden, int(experts),
                SC.DTYPES[dtype], self._parr(self._outs(recv)), recv_cap,
                self._parr(self._outs(route_pos)) if route_pos is not None else None,
                ctypes.c_void_p(SC._ptr(expert_counts)) if expert_counts is not None else None,
                ctypes.c_void_p(SC._ptr(recv_counts)) if recv_counts is not None else None, SC._stream(None)))
        self._call(go)

    def moe_combine(self, ys, y_rows, topk_idx, route_pos, topk_weight, experts, out, tokens, topk, hidden, dtype,
                    residual=None):
        """ys: every rank's registered expert-output rows [y_rows][hidden]; topk_idx, route_pos,
        topk_weight, out and residual (or None): this rank's own."""
        L = self._L

        def go():
            self._check(L.coll_moe_combine(
                self._h, self._parr(ys), y_rows, self._parr(self._outs(topk_idx)), self._parr(self._outs(route_pos)),
                self._parr(self._outs(topk_weight)),
                self._parr(self._outs(residual)) if residual is not None else None, tokens, topk, hidden,
                int(experts), SC.DTYPES[dtype], self._parr(self._outs(out)), SC._stream(None)))
        self._call(go)

    def close(self):
        for ptr in getattr(self, "_opened", []):
            self._L.sim_ipc_close(ctypes.c_void_p(ptr))
        self._opened = []
        super().close()
