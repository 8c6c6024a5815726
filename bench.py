"""Benchmark: effective HBM GB/s of the simulated-communicator collectives on one B200.

Workload (the DP gradient-bucket configuration): a communicator of p = 8 ranks in one GPU, each
rank holding a 25 Mi-element bucket (26,214,400 elements; 100 MiB fp32, 50 MiB bf16) of N(0, 1e-3)
values. One step runs every row of the hot path once on it:
  direct AllReduce AVG fp32 and bf16, ring AllReduce AVG fp32 and bf16 (1 MiB chunks),
  direct and ring Reduce SUM (root 2), Broadcast (root 2), ReduceScatter SUM, AllGather of the
  bucket's shards, equal All-to-All, and All-to-Allv of the bucket as 6,400 rows of 4,096 elements
  routed by a seeded top-2 / Zipf(1.1) router over 64 experts.
value = Σ (minimum HBM bytes of each call: every input read once, every output written once) /
device time of the step, summed over ranks (replicas) for N GPUs. The rows run back to back, so a
row's dirty L2 lines drain during the next row; each row is therefore also timed alone on a clean
L2 with its own write-back charged to it (per_op ms_attributed), and the direct rows are summed
on their own (direct_only). The ZeRO-shard (ReduceScatter of 256 Mi bf16 per rank, AllGather of
32 Mi-element bf16 shards) and MoE All-to-All (8,192 x 4,096 bf16 per rank, equal and top-2 /
Zipf counts) workloads are timed the same way in the `configs` block.

Prints one JSON line. ``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "effective HBM GB/s per collective vs ~8 TB/s peak (1×B200); oracle CPU GB/s"
P = 8
N_BUCKET = 26_214_400
HIDDEN = 4096
ROOT_RANK = 2
FALLBACK_HBM_GBS = 6650.0
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of a row's kernel, from an
# ncu capture of the current build, and the per-rank element count it was captured at.
NCU_TRAFFIC = {"allreduce_avg_fp32_ring": (2_184_816_640 + 1_417_508_352, 26_214_400)}
SPACER_CYCLES = 4_000_000  # ~2 ms of a spinning kernel ahead of a timed region


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="simcomm", choices=["simcomm", "reference"])
    ap.add_argument("--n", type=int, default=N_BUCKET, help="elements per rank (default: the 25 Mi bucket)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ops", default="", help="comma-separated substrings: run only the matching rows")
    ap.add_argument("--option", action="append", default=[], help="communicator option key=value")
    ap.add_argument("--sweep", action="store_true",
                    help="size/rank sweep with alpha-beta fits instead of the step (one GPU)")
    ap.add_argument("--sweep-ps", default="2,4,8,16,64")
    ap.add_argument("--sweep-max-bytes", type=int, default=1 << 30, help="largest per-rank message")
    ap.add_argument("--sweep-out", default="", help="write the sweep's markdown summary here")
    ap.add_argument("--moe", action="store_true",
                    help="time only the MoE dispatch and combine on the MoE workload (one GPU)")
    ap.add_argument("--no-moe", action="store_true", help="leave the MoE block out of the step's line")
    ap.add_argument("--moe-tokens", type=int, default=8192, help="tokens per rank of the MoE layer (--moe)")
    ap.add_argument("--no-configs", action="store_true",
                    help="leave the ZeRO-shard and MoE All-to-All blocks out of the step's line")
    ap.add_argument("--ceilings", action="store_true",
                    help="measure the HBM ceilings of the kernels' access patterns (load, store, copy, bulk "
                         "store) instead of the step (one GPU)")
    ap.add_argument("--ceilings-bytes", type=int, default=2 << 30, help="bytes each ceiling probe streams")
    ap.add_argument("--ceilings-out", default="", help="write the ceilings' markdown summary here")
    ap.add_argument("--no-attr", action="store_true",
                    help="skip the per-row timing with each row's write-back charged to it")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------------------------
# multi-GPU: independent replicas (one simulated communicator per GPU); the only cross-rank
# traffic is the timing plumbing below

def reduce_max(x, device=None):
    """Max of a host scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbps(world, bytes_per_step_per_rank, ms_per_step):
    """Whole-job throughput: every rank moves its step's bytes; the slowest rank sets the time."""
    return world * bytes_per_step_per_rank / (ms_per_step / 1e3) / 1e9


# ---------------------------------------------------------------------------------------------
# the step

def moe_rows_counts(n, p):
    """Rows of HIDDEN elements per (source, destination) for a bucket of n elements per rank."""
    from collective_communication_primitives_b200 import synth as S
    rows = n // HIDDEN
    tokens = rows // 2
    return S.moe_counts(p=p, tokens=tokens, experts=64, topk=2, zipf_s=1.1, hidden=1)


class Workload:
    def __init__(self, n, device):
        import numpy as np
        import torch

        from collective_communication_primitives_b200 import synth as S
        self.n, self.p = n, P
        self.m = n // P
        f32 = [S.normal(f"dp.fp32.rank{r}", n, 1e-3, "fp32") for r in range(P)]
        b16 = [S.normal(f"dp.bf16.rank{r}", n, 1e-3, "bf16") for r in range(P)]
        self.host_f32 = [torch.from_numpy(x).pin_memory() for x in f32]
        self.host_b16 = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in b16]
        self.x32 = [h.to(device) for h in self.host_f32]
        self.x16 = [h.to(device) for h in self.host_b16]
        self.ar32 = [torch.empty(n, dtype=torch.float32, device=device) for _ in range(P)]
        self.ar16 = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in range(P)]
        self.out32 = [torch.empty(n, dtype=torch.float32, device=device) for _ in range(P)]
        self.red = [None] * P
        self.red[ROOT_RANK] = torch.empty(n, dtype=torch.float32, device=device)
        self.rs = [torch.empty(self.m, dtype=torch.float32, device=device) for _ in range(P)]
        self.shards = [x[:self.m] for x in self.x32]
        rows = moe_rows_counts(n, P)
        self.counts_host = rows * HIDDEN
        self.counts = torch.from_numpy(self.counts_host).to(device)
        self.v_elems = int(self.counts_host.sum())
        self.v_send = [x[:int(self.counts_host[i].sum())] for i, x in enumerate(self.x32)]
        self.v_recv = [torch.empty(int(self.counts_host[:, j].sum()), dtype=torch.float32, device=device)
                       for j in range(P)]
        self.rows = rows

    def twin(self, device):
        """A second set of the buffers a host copy touches (the inputs and the AllReduce outputs), the
        rest shared, so that one step's copies can overlap another step's kernels."""
        import copy

        import torch
        t = copy.copy(self)
        t.x32 = [torch.empty_like(x) for x in self.x32]
        t.x16 = [torch.empty_like(x) for x in self.x16]
        t.ar32 = [torch.empty_like(x) for x in self.ar32]
        t.ar16 = [torch.empty_like(x) for x in self.ar16]
        t.shards = [x[:self.m] for x in t.x32]
        t.v_send = [x[:int(self.counts_host[i].sum())] for i, x in enumerate(t.x32)]
        return t


def build_step(comm, wl):
    """[(name, kernel, callable, effective bytes, kernel-model bytes)] for one step."""
    from collective_communication_primitives_b200 import bytemodel as BM
    n, p = wl.n, wl.p
    ops = []

    def add(name, kernel, fn, eff, kb):
        ops.append((name, kernel, fn, eff, kb))

    for algo in ("direct", "ring"):
        kern = "ring" if algo == "ring" else None
        add(f"allreduce_avg_fp32_{algo}", kern or "direct_reduce",
            lambda a=algo: comm.allreduce(wl.x32, wl.ar32, op="avg", algo=a),
            BM.direct_hbm_bytes("allreduce", p, n, 4),
            BM.ring_hbm_bytes("allreduce", p, n, 4) if algo == "ring" else BM.direct_hbm_bytes("allreduce", p, n, 4))
        add(f"allreduce_avg_bf16_{algo}", kern or "direct_reduce",
            lambda a=algo: comm.allreduce(wl.x16, wl.ar16, op="avg", algo=a),
            BM.direct_hbm_bytes("allreduce", p, n, 2),
            BM.ring_hbm_bytes("allreduce", p, n, 2, 4) if algo == "ring" else BM.direct_hbm_bytes("allreduce", p, n, 2))
        add(f"reduce_sum_fp32_{algo}", kern or "direct_reduce",
            lambda a=algo: comm.reduce(wl.x32, wl.red, ROOT_RANK, op="sum", algo=a),
            BM.direct_hbm_bytes("reduce", p, n, 4),
            BM.ring_hbm_bytes("reduce", p, n, 4) if algo == "ring" else BM.direct_hbm_bytes("reduce", p, n, 4))
        add(f"broadcast_fp32_{algo}", kern or "copy_engine",
            lambda a=algo: comm.broadcast(wl.x32, wl.out32, ROOT_RANK, algo=a),
            BM.direct_hbm_bytes("broadcast", p, n, 4),
            BM.ring_hbm_bytes("broadcast", p, n, 4) if algo == "ring" else BM.direct_hbm_bytes("broadcast", p, n, 4))
        add(f"reduce_scatter_sum_fp32_{algo}", kern or "direct_reduce",
            lambda a=algo: comm.reduce_scatter(wl.x32, wl.rs, op="sum", algo=a),
            BM.direct_hbm_bytes("reduce_scatter", p, n, 4),
            BM.ring_hbm_bytes("reduce_scatter", p, n, 4) if algo == "ring"
            else BM.direct_hbm_bytes("reduce_scatter", p, n, 4))
        add(f"allgather_fp32_{algo}", kern or "copy_engine",
            lambda a=algo: comm.allgather(wl.shards, wl.out32, algo=a),
            BM.direct_hbm_bytes("allgather", p, n, 4),
            BM.ring_hbm_bytes("allgather", p, n, 4) if algo == "ring" else BM.direct_hbm_bytes("allgather", p, n, 4))
        add(f"alltoall_fp32_{algo}", kern or "copy_engine",
            lambda a=algo: comm.alltoall(wl.x32, wl.out32, algo=a),
            BM.direct_hbm_bytes("alltoall", p, n, 4), BM.direct_hbm_bytes("alltoall", p, n, 4))
        add(f"alltoallv_fp32_{algo}", kern or "copy_engine",
            lambda a=algo: comm.alltoallv(wl.v_send, wl.v_recv, wl.counts, algo=a),
            BM.direct_hbm_bytes("alltoallv", p, 0, 4, moved_elems=wl.v_elems),
            BM.direct_hbm_bytes("alltoallv", p, 0, 4, moved_elems=wl.v_elems))
    return ops


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML every 20 ms while the timed region runs
    (nvidia-smi's command-line loop as a fallback)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.stop = threading.Event()
        self.thread = None

    def _nvml_loop(self):
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            self.stop.wait(0.02)
        pynvml.nvmlShutdown()

    def __enter__(self):
        try:
            import pynvml  # noqa: F401
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            time.sleep(0.05)
        except Exception:
            self.thread = None
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for _, _, rs in self.samples:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[0] for x in self.samples), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


def time_device(ops, steps, warmup, stream):
    """Warm up, then time exactly `steps` steps with events on the launching stream; also per-op
    events inside the timed region."""
    import torch
    for _ in range(warmup):
        for op in ops:
            op[2]()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops]
          for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    # keep the GPU busy while the host enqueues, so host-side call overhead never shows as idle time
    torch.cuda._sleep(SPACER_CYCLES)
    start.record(stream)
    for s in range(steps):
        for i, op in enumerate(ops):
            ev[s][i][0].record(stream)
            op[2]()
            ev[s][i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    per_op = [sum(ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(steps)) / steps for i in range(len(ops))]
    return total_ms, per_op


FLUSH_BYTES = 256 << 20  # twice the 126 MB L2: reading it evicts every line an earlier kernel left


class L2Flush:
    """A read-only pass over FLUSH_BYTES (a torch reduction): every line an earlier kernel left in
    L2, its dirty output lines included, is evicted, and a dirty line's write-back is paid inside
    this pass. It writes nothing large itself, so it leaves only clean lines behind."""

    def __init__(self, device):
        import torch
        self.buf = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.out = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self):
        import torch
        torch.sum(self.buf, 0, out=self.out)


def time_attributed(ops, steps, warmup, stream, flush):
    """Per-row device time with the row's own HBM write-back charged to it: each row runs on a clean
    L2 (after a flush) and is followed, inside its own event pair, by a flush that writes back the
    dirty lines the row left. The flush's own time on a clean L2 (median of as many runs) is
    subtracted. Returns (per-row ms, flush ms)."""
    import torch
    for _ in range(warmup):
        for op in ops:
            op[2]()
            flush()
    reps = max(steps, 5)
    fl = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops]
          for _ in range(steps)]
    torch.cuda.synchronize()
    torch.cuda._sleep(SPACER_CYCLES)
    flush()
    for e0, e1 in fl:
        e0.record(stream)
        flush()
        e1.record(stream)
    for s in range(steps):
        for i, op in enumerate(ops):
            ev[s][i][0].record(stream)
            op[2]()
            flush()
            ev[s][i][1].record(stream)
    torch.cuda.synchronize()
    flush_ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in fl)
    per_op = [sum(ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(steps)) / steps - flush_ms
              for i in range(len(ops))]
    return per_op, flush_ms


def time_e2e(comm, wl, make_ops, steps, warmup, stream, device):
    """The step through the public API with host buffers: every step copies all its inputs in from
    pinned host memory and both AllReduce results out, inside the timed region. Two buffer sets make
    a 2-deep pipeline: step k+1's host-to-device copies (one stream) and step k-1's device-to-host
    reads (another stream) overlap step k's kernels, ordered by events."""
    import torch
    sets = [wl, wl.twin(device)]
    ops = [make_ops(w) for w in sets]
    out_host32 = [torch.empty(wl.n, dtype=torch.float32).pin_memory() for _ in range(P)]
    out_host16 = [torch.empty(wl.n, dtype=torch.bfloat16).pin_memory() for _ in range(P)]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_h2d = [torch.cuda.Event() for _ in sets]
    ev_comp = [torch.cuda.Event() for _ in sets]
    ev_d2h = [torch.cuda.Event() for _ in sets]
    used = [False, False]

    def step(k):
        b = k % 2
        w = sets[b]
        with torch.cuda.stream(h2d_s):
            if used[b]:
                h2d_s.wait_event(ev_comp[b])  # the kernels that read these inputs are done
            for r in range(P):
                w.x32[r].copy_(wl.host_f32[r], non_blocking=True)
                w.x16[r].copy_(wl.host_b16[r], non_blocking=True)
            ev_h2d[b].record(h2d_s)
        stream.wait_event(ev_h2d[b])
        if used[b]:
            stream.wait_event(ev_d2h[b])  # the previous results in these buffers were read back
        for op in ops[b]:
            op[2]()
        ev_comp[b].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_comp[b])
            for r in range(P):
                out_host32[r].copy_(w.ar32[r], non_blocking=True)
                out_host16[r].copy_(w.ar16[r], non_blocking=True)
            ev_d2h[b].record(d2h_s)
        used[b] = True

    for k in range(warmup):
        step(k)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    h2d_s.wait_event(start)
    for k in range(warmup, warmup + steps):
        step(k)
    for b in range(2):
        if used[b]:
            stream.wait_event(ev_d2h[b])
    end.record(stream)
    torch.cuda.synchronize()
    h2d = P * wl.n * (4 + 2)
    d2h = P * wl.n * (4 + 2)
    return start.elapsed_time(end), h2d, d2h


def pcie_ceiling(device, nbytes=512 << 20, chunks=8, reps=3):
    """The host link's copy rates on this machine, the denominator of the e2e leg: pinned host memory to
    the device, the device to pinned host memory, and both directions at once on two streams (as the
    e2e pipeline runs them), each over `nbytes` in `chunks` copies, median of `reps`. GB/s per
    direction."""
    import torch
    n = nbytes // 4 // chunks
    h_in = [torch.empty(n, dtype=torch.float32).pin_memory() for _ in range(chunks)]
    h_out = [torch.empty(n, dtype=torch.float32).pin_memory() for _ in range(chunks)]
    d_in = [torch.empty(n, dtype=torch.float32, device=device) for _ in range(chunks)]
    d_out = [torch.zeros(n, dtype=torch.float32, device=device) for _ in range(chunks)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    cur = torch.cuda.current_stream()

    def run(h2d, d2h):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for c in range(chunks):
            if h2d:
                with torch.cuda.stream(s_in):
                    d_in[c].copy_(h_in[c], non_blocking=True)
            if d2h:
                with torch.cuda.stream(s_out):
                    h_out[c].copy_(d_out[c], non_blocking=True)
        cur.wait_stream(s_in)
        cur.wait_stream(s_out)
        e1.record(cur)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    out = {}
    for name, h2d, d2h in (("h2d_GBps", 1, 0), ("d2h_GBps", 0, 1), ("both_GBps_per_direction", 1, 1)):
        run(h2d, d2h)
        ms = statistics.median(run(h2d, d2h) for _ in range(reps))
        out[name] = round(chunks * n * 4 / (ms / 1e3) / 1e9, 1)
    return out


# ---------------------------------------------------------------------------------------------
# MoE dispatch and combine on the MoE workload

MOE = {"p": P, "tokens": 8192, "topk": 2, "experts": 64, "hidden": HIDDEN, "zipf_s": 1.1}


class MoeWorkload:
    """p ranks x 8192 tokens, top-2 of 64 experts with Zipf(1.1) popularity, 4096-wide bf16 rows;
    every receive buffer holds p*T*k rows (the worst case: all assignments to one rank)."""

    def __init__(self, device, tokens=None):
        import numpy as np
        import torch

        from collective_communication_primitives_b200 import synth as S
        p, T, k, E, H = P, tokens or MOE["tokens"], MOE["topk"], MOE["experts"], MOE["hidden"]
        self.p, self.T, self.k, self.E, self.H = p, T, k, E, H
        ids = S.moe_routes(p, T, E, k, MOE["zipf_s"], 0)
        ws = S.moe_gate_weights(p, T, k, 0)

        def bf16_rows(label, rows):
            return torch.from_numpy(S.normal(label, rows * H, 1.0, "bf16").view(np.int16)).view(torch.bfloat16) \
                .view(rows, H)

        self.host_x = [bf16_rows(f"moe.x.rank{i}", T).pin_memory() for i in range(p)]
        self.x = [h.to(device) for h in self.host_x]
        self.res = [bf16_rows(f"moe.res.rank{i}", T).to(device) for i in range(p)]
        self.idx = [torch.from_numpy(ids[i]).to(device) for i in range(p)]
        self.w = [torch.from_numpy(ws[i]).to(device) for i in range(p)]
        self.cap = p * T * k
        self.recv = [torch.empty(self.cap, H, dtype=torch.bfloat16, device=device) for _ in range(p)]
        self.pos = [torch.empty(T, k, dtype=torch.int32, device=device) for _ in range(p)]
        self.out = [torch.empty(T, H, dtype=torch.bfloat16, device=device) for _ in range(p)]
        self.recv_counts = torch.empty(p, dtype=torch.int64, device=device)
        self.expert_counts = torch.empty(p, E, dtype=torch.int64, device=device)
        self.col_rows = np.bincount((ids // (E // p)).reshape(-1), minlength=p)
        self.rank_rows = np.stack([np.bincount(ids[i].reshape(-1) // (E // p), minlength=p) for i in range(p)])


MOE_CPU_TOKENS = 2048  # the MoE CPU baseline: the first 2,048 tokens of every rank (a quarter of the layer)


def moe_cpu_baseline():
    """The oracle's dispatch + combine, as it stands and single-threaded, on the first MOE_CPU_TOKENS
    tokens of every rank of the same seeded layer (the generators are counter-based, so these are
    the GPU workload's own first tokens, routes and gate weights)."""
    import numpy as np

    import oracle as O
    from collective_communication_primitives_b200 import bytemodel as BM
    from collective_communication_primitives_b200 import synth as S
    p, T, k, E, H = P, MOE_CPU_TOKENS, MOE["topk"], MOE["experts"], MOE["hidden"]
    ids = S.moe_routes(p, T, E, k, MOE["zipf_s"], 0)
    ws = S.moe_gate_weights(p, T, k, 0)
    x = [S.normal(f"moe.x.rank{i}", T * H, 1.0, "bf16").reshape(T, H) for i in range(p)]
    res = [S.normal(f"moe.res.rank{i}", T * H, 1.0, "bf16").reshape(T, H) for i in range(p)]
    cap = int(np.bincount((ids // (E // p)).reshape(-1), minlength=p).max())
    t0 = time.perf_counter()
    d = O.moe_dispatch(x, list(ids), E, cap, "bf16")
    O.moe_combine(d["recv"], list(ids), list(ws), "bf16", E, residual=res, acc="slotfold")
    secs = time.perf_counter() - t0
    nbytes = BM.moe_dispatch_bytes(p, T, k, H, 2) + BM.moe_combine_bytes(p, T, k, H, 2, residual=True)
    return {"value": nbytes / secs / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"dispatch + combine of the first {T} tokens of each of the {p} ranks, single-threaded "
                      f"C++ oracle, {secs:.1f} s"}


def moe_ops(comm, mw):
    from collective_communication_primitives_b200 import bytemodel as BM
    p, T, k, H = mw.p, mw.T, mw.k, mw.H
    bd = BM.moe_dispatch_bytes(p, T, k, H, 2)
    bc = BM.moe_combine_bytes(p, T, k, H, 2, residual=True)
    return [
        ("moe_dispatch_bf16", "moe_dispatch (count, prefix sums, copy)",
         lambda: comm.moe_dispatch(mw.x, mw.idx, mw.E, mw.recv, route_pos=mw.pos, expert_counts=mw.expert_counts,
                                   recv_counts=mw.recv_counts), bd, bd),
        ("moe_combine_bf16", "moe_combine",
         lambda: comm.moe_combine(mw.recv, mw.idx, mw.pos, mw.w, mw.E, mw.out, residual=mw.res), bc, bc),
    ]


def moe_block(comm, mw, steps, warmup, stream, hbm, cpu=False):
    """Device time of the MoE dispatch and combine (behind a spacer, CUDA events) and their HBM
    roofline fractions."""
    import torch

    from collective_communication_primitives_b200 import synth as S
    ops = moe_ops(comm, mw)
    launches = []
    for op in ops:  # kernels one call launches (the comm's own count)
        l0 = comm.launch_count()
        op[2]()
        launches.append(comm.launch_count() - l0)
    torch.cuda.synchronize()
    _, per_op = time_device(ops, steps, warmup, stream)
    blk = {"workload": f"MoE layer, p={mw.p} ranks x {mw.T} tokens, top-{mw.k} of {mw.E} experts (Zipf 1.1), "
                       f"{mw.H}-wide bf16 rows", "max_recv_rows": int(mw.col_rows.max()),
           "rank_counts": S.count_matrix_stats(mw.rank_rows)}
    if cpu:
        blk["cpu_baseline"] = moe_cpu_baseline()
    for (name, kernel, _, eff, kb), ms, nl in zip(ops, per_op, launches):
        g = kb / (ms / 1e3) / 1e9
        blk[name] = {"ms": round(ms, 4), "GBps": round(g, 1), "frac_of_measured": round(g / hbm, 4),
                     "algorithmic_bytes": int(kb), "launches_per_call": int(nl)}
    return blk


def moe_main(args):
    import torch

    from collective_communication_primitives_b200 import simcomm as SC
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    mw = MoeWorkload("cuda:0", args.moe_tokens)
    comm = SC.SimComm(P)
    for kv in args.option:
        k, v = kv.split("=", 1)
        comm.set_option(k, int(v))
    hbm, peak_kind = peaks()
    ops = moe_ops(comm, mw)
    launches0 = comm.launch_count()
    with ClockSampler(0) as clk:
        total_ms, per_op = time_device(ops, args.steps, args.warmup, stream)
    launches = (comm.launch_count() - launches0) * args.steps // (args.steps + args.warmup)
    assert comm.async_error() == SC.OK
    eff = sum(o[3] for o in ops)
    ms = total_ms / args.steps
    i_dom = max(range(len(ops)), key=lambda i: per_op[i])
    name, kernel, _, _, kb = ops[i_dom]
    achieved = kb / (per_op[i_dom] / 1e3) / 1e9
    out = {"metric": METRIC, "value": round(eff / (ms / 1e3) / 1e9, 1), "unit": "GB/s", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16 rows, fp32 combine", "data": "synthetic",
           "config": {"workload": f"MoE dispatch + combine, p={P} ranks x {mw.T} tokens, top-{mw.k} of {mw.E} "
                                  f"experts (Zipf 1.1), {mw.H}-wide bf16 rows", "l2": "inputs larger than L2",
                      "options": args.option},
           "roofline": {"bound": "hbm", "kernel": f"{name} ({kernel})", "achieved": round(achieved, 1), "peak": hbm,
                        "unit": "GB/s", "frac": round(achieved / hbm, 4), "peak_source": peak_kind, "traffic": None,
                        "algorithmic_bytes_per_launch": int(kb), "ms_per_launch": round(per_op[i_dom], 4)},
           "per_op": {o[0]: {"ms": round(t, 4), "GBps": round(o[4] / (t / 1e3) / 1e9, 1),
                             "frac_of_measured": round(o[4] / (t / 1e3) / 1e9 / hbm, 4)} for o, t in zip(ops, per_op)},
           "gpu_launches": int(launches), "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = moe_cpu_baseline()
    print(json.dumps(out))
    comm.close()


# ---------------------------------------------------------------------------------------------
# The ZeRO-shard and MoE All-to-All workloads: every row timed with its own write-back charged

ZERO_N = 256 << 20            # bf16 elements per rank of the ZeRO partial-gradient tensor (512 MiB)
A2A_TOKENS = 8192             # tokens per rank of the MoE equal All-to-All


def device_normal(shape, sigma, gen, device):
    """Seeded N(0, sigma) bf16 drawn on the device (the values do not change a copy's or a
    reduction's time; the parity tests draw the same shapes from the counter-based host generator)."""
    import torch
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(0.0, sigma, generator=gen)
    return x.to(torch.bfloat16)


def zero_block(comm, steps, warmup, stream, flush, hbm, device):
    """ZeRO/FSDP shards: ReduceScatter of a 256 Mi-element bf16 partial gradient per rank (N(0,1e-2))
    to 32 Mi-element owner shards, then AllGather of 32 Mi-element bf16 parameter shards (N(0,0.02))
    back to 256 Mi per rank; direct and ring."""
    import torch

    from collective_communication_primitives_b200 import bytemodel as BM
    p, n = P, ZERO_N
    m = n // p
    gen = torch.Generator(device=device)
    gen.manual_seed(3)
    grads = [device_normal(n, 1e-2, gen, device) for _ in range(p)]
    params = [device_normal(m, 0.02, gen, device) for _ in range(p)]
    shards = [torch.empty(m, dtype=torch.bfloat16, device=device) for _ in range(p)]
    full = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in range(p)]
    ops = []
    for algo in ("direct", "ring"):
        ops.append((f"reduce_scatter_sum_bf16_{algo}", algo,
                    lambda a=algo: comm.reduce_scatter(grads, shards, op="sum", algo=a),
                    BM.direct_hbm_bytes("reduce_scatter", p, n, 2),
                    BM.ring_hbm_bytes("reduce_scatter", p, n, 2, 4) if algo == "ring"
                    else BM.direct_hbm_bytes("reduce_scatter", p, n, 2)))
        ops.append((f"allgather_bf16_{algo}", algo, lambda a=algo: comm.allgather(params, full, algo=a),
                    BM.direct_hbm_bytes("allgather", p, n, 2),
                    BM.ring_hbm_bytes("allgather", p, n, 2) if algo == "ring"
                    else BM.direct_hbm_bytes("allgather", p, n, 2)))
    blk = {"workload": f"ZeRO shards, p={p} ranks: ReduceScatter of {n} bf16 per rank to {m}-element shards; "
                       f"AllGather of {m}-element bf16 shards to {n} per rank",
           "l2": "each row on a clean L2 and followed, inside its own timing, by a read of 256 MiB that writes "
                 "back its dirty lines; that read's clean-L2 time subtracted"}
    blk.update(attributed_rows(ops, steps, warmup, stream, flush, hbm))
    del grads, params, shards, full
    torch.cuda.empty_cache()
    return blk


def moe_a2a_block(comm, steps, warmup, stream, flush, hbm, device):
    """MoE dispatch All-to-All: 8,192 tokens x 4,096 bf16 (N(0,1)) per rank, equal split (1,024
    tokens per destination), and the uneven All-to-Allv whose per-destination counts come from the
    seeded top-2 / Zipf(1.1) router over 64 experts (16,384 rows per rank); direct and ring."""
    import torch

    from collective_communication_primitives_b200 import bytemodel as BM
    from collective_communication_primitives_b200 import synth as S
    p, H = P, HIDDEN
    n = A2A_TOKENS * H
    gen = torch.Generator(device=device)
    gen.manual_seed(4)
    x = [device_normal(n, 1.0, gen, device) for _ in range(p)]
    y = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in range(p)]
    rows = S.moe_counts(p=p, tokens=A2A_TOKENS, experts=64, topk=2, zipf_s=1.1, hidden=1)
    counts_host = rows * H
    counts = torch.from_numpy(counts_host).to(device)
    v_send = [device_normal(int(counts_host[i].sum()), 1.0, gen, device) for i in range(p)]
    v_recv = [torch.empty(int(counts_host[:, j].sum()), dtype=torch.bfloat16, device=device) for j in range(p)]
    moved = int(counts_host.sum())
    ops = []
    for algo in ("direct", "ring"):
        ops.append((f"alltoall_bf16_{algo}", algo, lambda a=algo: comm.alltoall(x, y, algo=a),
                    BM.direct_hbm_bytes("alltoall", p, n, 2), BM.direct_hbm_bytes("alltoall", p, n, 2)))
        ops.append((f"alltoallv_bf16_{algo}", algo, lambda a=algo: comm.alltoallv(v_send, v_recv, counts, algo=a),
                    BM.direct_hbm_bytes("alltoallv", p, 0, 2, moved_elems=moved),
                    BM.direct_hbm_bytes("alltoallv", p, 0, 2, moved_elems=moved)))
    blk = {"workload": f"MoE dispatch All-to-All, p={p} ranks x {A2A_TOKENS} tokens x {H} bf16: equal split "
                       f"({A2A_TOKENS // p} tokens per destination) and All-to-Allv on top-2 / Zipf(1.1) counts over "
                       f"64 experts", "alltoallv_rows": dict(S.count_matrix_stats(rows), total=int(rows.sum())),
           "l2": "as zero_shards"}
    blk.update(attributed_rows(ops, steps, warmup, stream, flush, hbm))
    del x, y, v_send, v_recv
    torch.cuda.empty_cache()
    return blk


def attributed_rows(ops, steps, warmup, stream, flush, hbm):
    per_op, flush_ms = time_attributed(ops, steps, warmup, stream, flush)
    rows = {}
    for (name, algo, _, eff, kb), ms in zip(ops, per_op):
        rows[name] = {"ms": round(ms, 4), "effective_GBps": round(eff / (ms / 1e3) / 1e9, 1),
                      "kernel_GBps": round(kb / (ms / 1e3) / 1e9, 1),
                      "frac_of_measured_peak": round(kb / (ms / 1e3) / 1e9 / hbm, 4),
                      "frac_of_nominal_8TBps": round(kb / (ms / 1e3) / 1e9 / 8000.0, 4),
                      "minimum_bytes": int(eff), "model_bytes": int(kb)}
    return {"rows": rows, "flush_ms": round(flush_ms, 4)}


# ---------------------------------------------------------------------------------------------
# the oracle as a CPU baseline (and as the reference arm)

def oracle_inputs(n):
    """The step's inputs for the oracle, from the same seeded recipe, generated on the host."""
    from collective_communication_primitives_b200 import synth as S
    p = P
    x32 = [S.normal(f"dp.fp32.rank{r}", n, 1e-3, "fp32") for r in range(p)]
    x16 = [S.normal(f"dp.bf16.rank{r}", n, 1e-3, "bf16") for r in range(p)]
    counts = moe_rows_counts(n, p) * HIDDEN
    vsend = [x32[i][:int(counts[i].sum())] for i in range(p)]
    return {"n": n, "x32": x32, "x16": x16, "counts": counts, "vsend": vsend}


def oracle_step(inp):
    """Run the oracle over every row of the step once; returns (seconds, effective bytes)."""
    import oracle as O
    from collective_communication_primitives_b200 import bytemodel as BM
    p, n = P, inp["n"]
    m = n // p
    x32, x16, counts, vsend = inp["x32"], inp["x16"], inp["counts"], inp["vsend"]
    t0 = time.perf_counter()
    O.allreduce(x32, "fp32", "avg", acc="rankfold")
    O.allreduce(x16, "bf16", "avg", acc="rankfold")
    O.ring_allreduce(x32, "fp32", "avg")
    O.ring_allreduce(x16, "bf16", "avg")
    O.reduce(x32, "fp32", "sum", ROOT_RANK, acc="rankfold")
    O.ring_reduce(x32, "fp32", "sum", ROOT_RANK)
    O.broadcast(x32[ROOT_RANK], p, "fp32", ROOT_RANK)
    O.ring_broadcast(x32[ROOT_RANK], p, "fp32", ROOT_RANK)
    O.reduce_scatter(x32, "fp32", "sum", acc="rankfold")
    O.ring_reduce_scatter(x32, "fp32", "sum")
    O.allgather([x[:m] for x in x32], "fp32")
    O.ring_allgather([x[:m] for x in x32], "fp32")
    O.alltoall(x32, "fp32")
    O.ring_alltoall(x32, "fp32")
    O.alltoallv(vsend, counts, "fp32")
    O.alltoallv(vsend, counts, "fp32")
    secs = time.perf_counter() - t0
    eff = 2 * (BM.direct_hbm_bytes("allreduce", p, n, 4) + BM.direct_hbm_bytes("allreduce", p, n, 2) +
               BM.direct_hbm_bytes("reduce", p, n, 4) + BM.direct_hbm_bytes("broadcast", p, n, 4) +
               BM.direct_hbm_bytes("reduce_scatter", p, n, 4) + BM.direct_hbm_bytes("allgather", p, n, 4) +
               BM.direct_hbm_bytes("alltoall", p, n, 4) +
               BM.direct_hbm_bytes("alltoallv", p, 0, 4, moved_elems=int(counts.sum())))
    return secs, eff


CPU_SAMPLE_N = N_BUCKET             # the CPU baseline: one full step (about 10-20 s of CPU work)
REF_SAMPLE_N = N_BUCKET // 8        # one reference-arm step: 1/8 of the bucket


def oracle_slices(inp, parts):
    """Cut the step's inputs into `parts` independent steps on contiguous element ranges of every
    rank's bucket (each a multiple of p * 64 elements), the All-to-Allv counts redrawn per range."""
    n, unit = inp["n"], P * 64
    per = max(unit, (n // parts) // unit * unit)
    cuts = [min(n, i * per) for i in range(parts)] + [n]
    out = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        if hi <= lo:
            continue
        x32 = [x[lo:hi] for x in inp["x32"]]
        counts = moe_rows_counts(hi - lo, P) * HIDDEN
        out.append({"n": hi - lo, "x32": x32, "x16": [x[lo:hi] for x in inp["x16"]], "counts": counts,
                    "vsend": [x32[i][:int(counts[i].sum())] for i in range(P)]})
    return out


def oracle_step_threads(inp, threads):
    """The oracle step run by `threads` host threads at once, each on its own slice of the bucket
    (the oracle's C calls release the interpreter lock); returns (wall seconds, effective bytes,
    threads used)."""
    parts = oracle_slices(inp, threads)
    res = [None] * len(parts)
    go = threading.Barrier(len(parts) + 1)

    def work(i):
        go.wait()
        res[i] = oracle_step(parts[i])

    ts = [threading.Thread(target=work, args=(i,)) for i in range(len(parts))]
    for t in ts:
        t.start()
    go.wait()
    t0 = time.perf_counter()
    for t in ts:
        t.join()
    return time.perf_counter() - t0, sum(r[1] for r in res), len(parts)


def host_threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def cpu_baseline():
    """The oracle as it stands, timed twice on the same full-bucket step: single-threaded, and on
    every host core with one contiguous element range of each rank's bucket per thread."""
    inp = oracle_inputs(CPU_SAMPLE_N)
    secs, eff = oracle_step(inp)
    mt_secs, mt_eff, used = oracle_step_threads(inp, host_threads())
    return {"value": eff / secs / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"one step of every row on the full bucket (p={P}, n={CPU_SAMPLE_N} per rank), "
                      f"single-threaded C++ oracle, {secs:.1f} s",
            "all_cores": {"value": mt_eff / mt_secs / 1e9, "unit": "GB/s", "cores": used,
                          "sample": f"the same step cut into {used} contiguous element ranges of every rank's "
                                    f"bucket, one oracle step per host thread, all at once, {mt_secs:.1f} s wall"}}


# The rows of one step, in the order build_step() issues them (the oracle step runs the same rows).
STEP_ROWS = tuple(f"{op}_{algo}" for algo in ("direct", "ring") for op in (
    "allreduce_avg_fp32", "allreduce_avg_bf16", "reduce_sum_fp32", "broadcast_fp32", "reduce_scatter_sum_fp32",
    "allgather_fp32", "alltoall_fp32", "alltoallv_fp32"))


def step_config(n, world, rows, options):
    """The `config` of the step's JSON line, shared by this arm and the reference arm."""
    from collective_communication_primitives_b200 import synth as S
    v_stats = dict(S.count_matrix_stats(moe_rows_counts(n, P)), unit=f"rows of {HIDDEN} elements")
    return {"workload": f"DP gradient bucket, p={P} ranks x {n} elements per rank, every hot-path row "
                        f"(direct and ring) per step", "p": P, "n_per_rank": n,
            "chunk_bytes": 1 << 20, "l2": "inputs larger than L2 (100 MiB per rank fp32)",
            "ops": rows, "alltoallv_counts": v_stats, "options": options, "parallelism": f"replicas x{world}"}


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = oracle_inputs(REF_SAMPLE_N)
    for _ in range(args.warmup):
        oracle_step(inp)
    tot_s, tot_b = 0.0, 0
    for _ in range(args.steps):
        s, b = oracle_step(inp)
        tot_s += s
        tot_b += b
    v = tot_b / tot_s / 1e9
    sample = (f"each step: every row of the step on the first {REF_SAMPLE_N} elements of each rank's bucket (1/8 of "
              f"the workload; the counter-based inputs are the GPU run's own), single-threaded C++ oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32+bf16 (fp32 accumulate)", "data": "synthetic",
        "config": step_config(N_BUCKET, args.gpus, list(STEP_ROWS), args.option),
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ---------------------------------------------------------------------------------------------
# size / rank sweep: latency, algbw, busbw and alpha-beta fits per (op, path, p)

SWEEP_OPS = ("allreduce", "reduce", "broadcast", "reduce_scatter", "allgather", "alltoall")
SWEEP_CAP_BYTES = 64 << 30  # total device memory a point may hold


def sweep(args):
    import numpy as np
    import torch

    from collective_communication_primitives_b200 import bytemodel as BM
    from collective_communication_primitives_b200 import simcomm as SC
    torch.cuda.set_device(0)
    dev = "cuda:0"
    stream = torch.cuda.current_stream()
    sizes = []
    b = 1024
    while b <= args.sweep_max_bytes:
        sizes.append(b)
        b *= 4
    rows = []
    for p in [int(x) for x in args.sweep_ps.split(",")]:
        comm = SC.SimComm(p)
        algos = ("direct", "ring", "rd", "hd", "tree", "dbtree", "ll", "rd_ll", "tree_ll", "dbtree_ll") \
            if p & (p - 1) == 0 else ("direct", "ring", "tree", "dbtree", "ll", "tree_ll", "dbtree_ll")
        for algo in algos:
            for nbytes in sizes:
                n = max(p, (nbytes // 4) // p * p)     # int32 elements, divisible by p
                hold = 2 * p * n * 4 + {"direct": 0, "ring": 1, "rd": 2, "hd": 1, "tree": 1, "dbtree": 1, "ll": 0,
                                        "rd_ll": 0, "tree_ll": 0, "dbtree_ll": 0}[algo] * p * n * 4
                if hold > SWEEP_CAP_BYTES:
                    continue
                if algo == "ll" and p * (2 * p - 3) * -(-n // p) * 8 > (256 << 20):
                    continue  # the LL protocol's receive slots are capped (small messages only)
                if algo == "rd_ll" and (n > (1 << 20) // p or p * p.bit_length() * n * 8 > (256 << 20)):
                    continue  # registers of one resident grid hold the vector (small messages only)
                if algo in ("tree_ll", "dbtree_ll") and p * 3 * n * 8 > (256 << 20):
                    continue  # the LL protocol's receive slots are capped (small messages only)
                x = [torch.randint(-2**24, 2**24, (n,), dtype=torch.int32, device=dev) for _ in range(p)]
                y = [torch.empty(n, dtype=torch.int32, device=dev) for _ in range(p)]
                m = n // p
                calls = {
                    "allreduce": lambda: comm.allreduce(x, y, op="sum", algo=algo),
                    "reduce": lambda: comm.reduce(x, y, 0, op="sum", algo=algo),
                    "broadcast": lambda: comm.broadcast(x, y, 0, algo=algo),
                    "reduce_scatter": lambda: comm.reduce_scatter(x, [t[:m] for t in y], op="sum", algo=algo),
                    "allgather": lambda: comm.allgather([t[:m] for t in x], y, algo=algo),
                    "alltoall": lambda: comm.alltoall(x, y, algo=algo),
                }
                for op in (SWEEP_OPS if algo in ("direct", "ring") else ("allreduce",)):
                    f = calls[op]
                    for _ in range(3):
                        f()
                    torch.cuda.synchronize()
                    # 10 back-to-back calls enqueued behind a spinning kernel: device time per call,
                    # without host-side call overhead (which would otherwise leave the GPU idle)
                    reps = 10
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    torch.cuda._sleep(SPACER_CYCLES)
                    e0.record(stream)
                    for _ in range(reps):
                        f()
                    e1.record(stream)
                    e1.synchronize()
                    ms = e0.elapsed_time(e1) / reps
                    msg = n * 4  # per-rank message: the AllReduce in/out, ReduceScatter input, AllGather output
                    hbm = BM.direct_hbm_bytes(op, p, n, 4)
                    algbw = msg / (ms / 1e3) / 1e9
                    rows.append({"p": p, "algo": algo, "op": op, "bytes_per_rank": msg, "ms": ms,
                                 "algbw_GBps": algbw, "busbw_GBps": algbw * BM.busbw_factor(op, p),
                                 "hbm_GBps": hbm / (ms / 1e3) / 1e9,
                                 "l2_resident": p * msg * 2 < 2 * 126e6})
                    assert comm.async_error() == SC.OK
                del x, y
                torch.cuda.empty_cache()
        comm.close()
    fits = []
    for p in sorted({r["p"] for r in rows}):
        for algo in ("direct", "ring", "rd", "hd", "tree", "dbtree", "ll", "rd_ll", "tree_ll", "dbtree_ll"):
            for op in SWEEP_OPS:
                pts = [r for r in rows if r["p"] == p and r["algo"] == algo and r["op"] == op]
                if len(pts) < 3:
                    continue
                mb = np.array([r["bytes_per_rank"] for r in pts], float)
                t = np.array([r["ms"] * 1e-3 for r in pts])
                A = np.stack([np.ones_like(mb), mb], axis=1)
                (alpha, inv_beta), *_ = np.linalg.lstsq(A, t, rcond=None)
                fit = {"p": p, "algo": algo, "op": op, "alpha_us": alpha * 1e6,
                       "beta_GBps": (1.0 / inv_beta) / 1e9 if inv_beta > 0 else None}
                if algo == "ring" and op == "allreduce" and p > 1:
                    # the ring model: T = 2(p-1) alpha_hop + 2(p-1)/p * m / beta
                    A2 = np.stack([np.full_like(mb, 2 * (p - 1)), 2 * (p - 1) / p * mb], axis=1)
                    (ah, ib), *_ = np.linalg.lstsq(A2, t, rcond=None)
                    fit["ring_alpha_hop_us"] = ah * 1e6
                    fit["ring_beta_GBps"] = (1.0 / ib) / 1e9 if ib > 0 else None
                fits.append(fit)
    for r in rows:
        print(json.dumps({"sweep_point": r}))
    for f in fits:
        print(json.dumps({"sweep_fit": f}))
    if args.sweep_out:
        write_sweep_md(args.sweep_out, rows, fits)


def write_sweep_md(path, rows, fits):
    lines = ["# Size / rank sweep: latency, bandwidth and alpha-beta fits", "",
             "int32 SUM data, per-rank message m = n*4 bytes (the AllReduce buffer, the ReduceScatter input,",
             "the AllGather output, the All-to-All send buffer); 10 back-to-back calls after 3 warm-ups, enqueued",
             "behind a spinning kernel and timed with CUDA events (device time per call, launch gaps included). algbw = m / t; busbw = algbw x the bus-bandwidth factor; hbm = minimum HBM bytes of the",
             "call / t. Points whose p*m*2 fits in ~2x the 126 MB L2 are marked L2.", "",
             "## Fits: t = alpha + m / beta (least squares over the sizes of each line)", "",
             "| p | path | op | alpha (us) | beta (GB/s of m) | ring model: alpha per hop (us) | ring model: beta (GB/s) |",
             "|---:|---|---|---:|---:|---:|---:|"]
    def num(x, fmt):
        return format(x, fmt) if x is not None else "n/a"
    for f in fits:
        lines.append(f"| {f['p']} | {f['algo']} | {f['op']} | {num(f['alpha_us'], '.2f')} | "
                     f"{num(f['beta_GBps'], '.1f')} | {num(f.get('ring_alpha_hop_us'), '.2f')} | "
                     f"{num(f.get('ring_beta_GBps'), '.1f')} |")
    lines += ["", "## Points", "", "| p | path | op | m (bytes) | t (us) | algbw GB/s | busbw GB/s | HBM GB/s | L2 |",
              "|---:|---|---|---:|---:|---:|---:|---:|---|"]
    for r in rows:
        lines.append(f"| {r['p']} | {r['algo']} | {r['op']} | {r['bytes_per_rank']} | {r['ms']*1e3:.1f} | "
                     f"{r['algbw_GBps']:.1f} | {r['busbw_GBps']:.1f} | {r['hbm_GBps']:.1f} | "
                     f"{'L2' if r['l2_resident'] else ''} |")
    with open(path, "w") as fh:
        fh.write("\n".join(lines) + "\n")


# ---------------------------------------------------------------------------------------------
# HBM ceilings of the access patterns the kernels use

def ceilings(args):
    """Each access pattern of the library's kernels alone (sim_hbm_probe) over a buffer 16x the L2,
    at several CTAs per SM (the 1:8 bulk fan-out reads an eighth of it and writes it 8 times); plus
    torch's copy_ (the measured peak's own method) and fill_ for reference.
    GB/s counts every byte read plus every byte written, best of 5 launches after 2 warm-ups."""
    import torch

    from collective_communication_primitives_b200 import simcomm as SC
    torch.cuda.set_device(0)
    dev = "cuda:0"
    nb = args.ceilings_bytes // (16 << 10) * (16 << 10)
    src = torch.ones(nb // 4, dtype=torch.float32, device=dev)
    dst = torch.empty(nb // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    hbm, peak_kind = peaks()

    flush = L2Flush(dev)

    def timed(fn, reps=5):
        """Best of `reps`, each on a clean L2 and charged with its own write-back (the flush after it
        inside the events, the flush's clean-L2 time subtracted): the timing of the attributed rows."""
        for _ in range(2):
            fn()
        fl, best = [], None
        for _ in range(reps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            flush()
            e1.record(stream)
            e1.synchronize()
            fl.append(e0.elapsed_time(e1))
        f_ms = statistics.median(fl)
        for _ in range(reps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            flush()
            e1.record(stream)
            e1.synchronize()
            ms = e0.elapsed_time(e1) - f_ms
            best = ms if best is None else min(best, ms)
        return best

    rows = []
    with ClockSampler(0) as clk:
        for kind in ("load", "store", "copy", "bulk_store"):
            moved = nb * (2 if kind == "copy" else 1)
            for cps in (0, 1, 2, 4, 8):
                ms = timed(lambda: SC.hbm_probe(kind, dst if kind != "load" else None,
                                                src if kind in ("load", "copy") else None, nb, cps))
                rows.append({"pattern": kind, "ctas_per_sm": cps, "bytes_moved": moved, "ms": round(ms, 4),
                             "GBps": round(moved / (ms / 1e3) / 1e9, 1)})
        for fan_nb in (nb // 8 // (32 << 10) * (32 << 10), 100 << 20):  # an eighth of the buffer; the DP bucket
            for cps in (1, 2, 3):
                ms = timed(lambda: SC.hbm_probe("bulk_fanout", dst, src, fan_nb, cps))
                rows.append({"pattern": f"bulk_fanout {fan_nb >> 20} MiB", "ctas_per_sm": cps,
                             "bytes_moved": 9 * fan_nb, "ms": round(ms, 4),
                             "GBps": round(9 * fan_nb / (ms / 1e3) / 1e9, 1)})
        ms = timed(lambda: dst.copy_(src))
        rows.append({"pattern": "torch copy_", "ctas_per_sm": None, "bytes_moved": 2 * nb, "ms": round(ms, 4),
                     "GBps": round(2 * nb / (ms / 1e3) / 1e9, 1)})
        ms = timed(lambda: dst.fill_(2.0))
        rows.append({"pattern": "torch fill_", "ctas_per_sm": None, "bytes_moved": nb, "ms": round(ms, 4),
                     "GBps": round(nb / (ms / 1e3) / 1e9, 1)})
    best = {}
    for r in rows:
        if r["pattern"] not in best or r["GBps"] > best[r["pattern"]]["GBps"]:
            best[r["pattern"]] = r
    out = {"ceilings": {k: {"GBps": v["GBps"], "ctas_per_sm": v["ctas_per_sm"], "frac_of_measured": round(v["GBps"] / hbm, 4)}
                        for k, v in best.items()},
           "peak": hbm, "peak_source": peak_kind, "bytes": nb, "rows": rows, "clocks": clk.summary()}
    print(json.dumps(out))
    if args.ceilings_out:
        lines = [f"| pattern | CTAs per SM | GB/s (read + written) | of measured {hbm:.1f} GB/s |",
                 "|---|---:|---:|---:|"]
        for r in rows:
            cps = {None: "-", 0: "one pass"}.get(r["ctas_per_sm"], r["ctas_per_sm"])
            lines.append(f"| {r['pattern']} | {cps} | {r['GBps']:.1f} | "
                         f"{r['GBps'] / hbm:.3f} |")
        with open(args.ceilings_out, "w") as fh:
            fh.write("\n".join(lines) + "\n")


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.sweep:
        sweep(args)
        return
    if args.moe:
        moe_main(args)
        return
    if args.ceilings:
        ceilings(args)
        return
    import torch
    import torch.distributed as dist

    from collective_communication_primitives_b200 import simcomm as SC

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    device = f"cuda:{local}"
    stream = torch.cuda.current_stream()

    wl = Workload(args.n, device)
    comm = SC.SimComm(P)
    comm.set_option("chunk_bytes", 1 << 20)
    for kv in args.option:
        k, v = kv.split("=", 1)
        comm.set_option(k, int(v))
    keys = [k for k in args.ops.split(",") if k]

    def make_ops(w):
        return [o for o in build_step(comm, w) if not keys or any(k in o[0] for k in keys)]

    ops = make_ops(wl)
    eff_per_step = sum(o[3] for o in ops)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = comm.launch_count()
    with ClockSampler(local) as clk:
        total_ms, per_op = time_device(ops, args.steps, args.warmup, stream)
    launches = comm.launch_count() - launches0 - args.warmup * len(ops)
    clocks = clk.summary()
    torch.cuda.synchronize()
    if world > 1:
        total_ms = reduce_max(total_ms, device)
        dist.barrier()

    e2e = None
    if not args.no_e2e:
        # as many timed steps as the device timing: the pipeline's fill (the first step's copies in)
        # and drain (the last step's results out) are paid once per run, not per step
        e_steps = args.steps
        e_ms, h2d, d2h = time_e2e(comm, wl, make_ops, e_steps, 1, stream, device)
        if world > 1:
            e_ms = reduce_max(e_ms, device)
        link = pcie_ceiling(device)
        # the copies alone, both directions at once at the link's measured rate: the e2e step's floor
        floor_ms = max(h2d, d2h) / (link["both_GBps_per_direction"] * 1e9) * 1e3
        e2e = {"value": job_gbps(world, eff_per_step, e_ms / e_steps), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms / e_steps, 3),
               "steps": e_steps, "host_link": link, "copy_floor_ms_per_step": round(floor_ms, 3),
               "frac_of_copy_floor": round(floor_ms / (e_ms / e_steps), 4),
               "pipeline": "2 buffer sets: step k+1's host-to-device copies and step k-1's device-to-host "
                           "reads overlap step k's kernels; the first step's copies in and the last step's "
                           "reads out are inside the timed region"}

    hbm, peak_kind = peaks()
    ms_per_step = total_ms / args.steps
    value = job_gbps(world, eff_per_step, ms_per_step)
    # Each row again, on a clean L2 and charged with its own write-back (the back-to-back times above
    # let a row's dirty lines drain during the next row).
    flush = L2Flush(device)
    attr = None
    if not args.no_attr:
        attr, flush_ms = time_attributed(ops, args.steps, args.warmup, stream, flush)
    per_op_json = {}
    for i, ((name, kernel, _, eff, kb), ms) in enumerate(zip(ops, per_op)):
        per_op_json[name] = {"ms": round(ms, 4), "effective_GBps": round(eff / (ms / 1e3) / 1e9, 1),
                             "kernel_GBps": round(kb / (ms / 1e3) / 1e9, 1),
                             "frac_of_measured_peak": round(kb / (ms / 1e3) / 1e9 / hbm, 4)}
        if attr:
            a = attr[i]
            per_op_json[name].update({"ms_attributed": round(a, 4), "kernel_GBps_attributed": round(kb / (a / 1e3) / 1e9, 1),
                                      "frac_attributed": round(kb / (a / 1e3) / 1e9 / hbm, 4)})
    # The direct rows alone (the collective's minimum bytes over the direct kernels' time).
    d_idx = [i for i, o in enumerate(ops) if o[0].endswith("_direct")]
    direct_only = None
    if d_idx:
        d_bytes = sum(ops[i][3] for i in d_idx)
        d_ms = sum(per_op[i] for i in d_idx)
        direct_only = {"value": round(job_gbps(world, d_bytes, d_ms), 1), "unit": "GB/s",
                       "ms_per_step": round(d_ms, 4), "rows": len(d_idx),
                       "timing": "back to back, as the step"}
        if attr:
            a_ms = sum(attr[i] for i in d_idx)
            direct_only.update({"value_attributed": round(job_gbps(world, d_bytes, a_ms), 1),
                                "ms_per_step_attributed": round(a_ms, 4)})
    # The dominant kernel: each row is one launch of one kernel, so the row with the largest share
    # of the step's device time names it. achieved = that kernel's algorithmic bytes per launch (its
    # byte model: the minimum for direct rows; for ring rows the schedule's hop traffic, every hop
    # reading a partial and an input and writing a partial or an output, which ncu's DRAM counters
    # confirm at this size) over its average launch time measured above with CUDA events. The
    # collective's minimum bytes (any schedule) are reported beside it.
    i_dom = max(range(len(ops)), key=lambda i: per_op[i])
    name, kernel, _, eff, kb = ops[i_dom]
    d_ms = per_op[i_dom]
    achieved = kb / (d_ms / 1e3) / 1e9
    traffic = None
    if name in NCU_TRAFFIC and args.n in (NCU_TRAFFIC[name][1], N_BUCKET):
        t_bytes, t_n = NCU_TRAFFIC[name]
        traffic = int(t_bytes * args.n / t_n)
    roofline = {"bound": "hbm", "kernel": f"{name} ({kernel})", "achieved": round(achieved, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(achieved / hbm, 4), "peak_source": peak_kind,
                "traffic": traffic, "algorithmic_bytes_per_launch": int(kb),
                "minimum_bytes_per_launch": int(eff),
                "share_of_step": round(d_ms / sum(per_op), 4), "ms_per_launch": round(d_ms, 4)}
    # The four direct kernels the throughput target names (>= 80% of the ~8 TB/s nominal peak at
    # >= 64 MB per rank), on every workload that runs them: each row charged with its own write-back
    # where that timing ran (else back to back).
    target = {}
    for i, ((nm, kernel, _, eff, kb), ms) in enumerate(zip(ops, per_op)):
        if nm in ("allreduce_avg_fp32_direct", "allreduce_avg_bf16_direct", "reduce_scatter_sum_fp32_direct",
                  "allgather_fp32_direct", "alltoall_fp32_direct"):
            t = attr[i] if attr else ms
            g = kb / (t / 1e3) / 1e9
            target["dp_bucket." + nm] = {"GBps": round(g, 1), "frac_of_measured": round(g / hbm, 4),
                                         "frac_of_nominal_8TBps": round(g / 8000.0, 4),
                                         "back_to_back_GBps": round(kb / (ms / 1e3) / 1e9, 1)}
    configs = {}
    if not args.no_configs and not args.ops and args.n == N_BUCKET:
        configs["zero_shards"] = zero_block(comm, args.steps, args.warmup, stream, flush, hbm, device)
        configs["moe_alltoall"] = moe_a2a_block(comm, args.steps, args.warmup, stream, flush, hbm, device)
        for cname, blk in configs.items():
            for nm, row in blk["rows"].items():
                if nm.endswith("_direct") and nm.split("_")[0] in ("reduce", "allgather", "alltoall"):
                    target[f"{cname}.{nm}"] = {"GBps": row["kernel_GBps"], "frac_of_measured": row["frac_of_measured_peak"],
                                               "frac_of_nominal_8TBps": row["frac_of_nominal_8TBps"]}
    del flush

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32+bf16 (fp32 accumulate)", "data": "synthetic",
        "config": step_config(args.n, world, [o[0] for o in ops], args.option),
        "roofline": roofline,
        "direct_only": direct_only,
        "target_direct": target,
        "per_op": per_op_json,
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if e2e:
        out["e2e"] = e2e
    if attr:
        out["attribution"] = {"flush_bytes": FLUSH_BYTES, "flush_ms_clean": round(flush_ms, 4),
                              "how": "per row: clean L2, the row, a read of flush_bytes that writes back the "
                                     "row's dirty lines, all inside the row's events; the read's clean-L2 time "
                                     "subtracted"}
    if configs:
        out["configs"] = configs
    if not args.no_moe and not args.ops:
        mw = MoeWorkload(device)
        out["moe"] = moe_block(comm, mw, max(3, args.steps // 2), args.warmup, stream, hbm,
                               cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline))
        del mw
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(out))
    comm.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
