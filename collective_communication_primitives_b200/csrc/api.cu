// Host side of the C ABI declared in include/simcomm.h: communicator lifecycle, options,
// argument validation, asynchronous error state and dispatch to the kernels.
//
// Citations name "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives)
// as [Atlas] and "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All"
// (charlestar.github.io/2026/08/20/gpu-collective-communication) as [Primer].
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cctype>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "internal.h"
#include "simcomm.h"

using namespace simcomm;

// One traced call: its record and the two events that bracket its kernels on the caller's stream.
struct TraceSlot {
    sim_comm_trace_record_t rec{};
    cudaEvent_t ev0 = nullptr, ev1 = nullptr;
    bool timed = false;
};
constexpr size_t kTraceCap = 4096;

struct sim_comm {
    int p = 0;
    int rank = -1;                  // a rank view: the one rank of p processes this handle computes for
    int device = 0;
    int num_sms = 0;
    DevState* dstate = nullptr;     // device scratch header
    uint32_t* host_words = nullptr; // host-mapped: [0] status mirror, [1] abort flag
    uint32_t* dev_words = nullptr;  // device alias of host_words
    unsigned long long* flags = nullptr;  // ring chunk flags
    size_t flags_cap = 0;           // elements
    char* stage = nullptr;          // ring partial buffers
    size_t stage_cap = 0;           // bytes
    unsigned long long* ll = nullptr;  // LL receive slots
    size_t ll_cap = 0;              // bytes
    uint32_t ll_epoch = 0;          // LL tags: slot q of call e carries e * 128 + 1 + q
    int ll_ctas_max = 0;
    char* moe = nullptr;            // MoE dispatch counting and prefix scratch
    size_t moe_cap = 0;             // bytes
    int32_t* moe_acc = nullptr;     // fused MoE dispatch: per-(rank, expert) totals, zero between calls
    size_t moe_acc_cap = 0;         // elements
    uint32_t epoch = 0;
    long long chunk_bytes = 1 << 20;
    long long ring_ctas = 0;
    long long timeout_ns = 2000000000LL;
    long long fault_skip_rank = -1;
    long long copy_variant = -1;
    long long copy_order = -1;
    long long direct_pack = 0;
    long long direct_ctas_per_sm = 16;
    long long l2_hint = -1;
    long long ring_task_bytes = 0;  // bytes of the wire type one ring / tree task moves; 0 = by message size
    long long moe_tma = 0;          // MoE dispatch copy: 0 loads and stores (faster, measured), 1 bulk copies
    long long moe_fused = 1;        // MoE dispatch: 1 one cooperative kernel, 0 three kernels
    unsigned long long launches = 0;
    int ring_ctas_max = 0;
    bool capturing = false;               // the current call's stream is being captured into a graph
    bool captured_any = false;            // some call was captured: graphs may hold scratch pointers
    std::vector<void*> retired;           // scratch replaced after a capture, freed at destroy
    std::vector<std::pair<int32_t*, size_t>> retired_acc;  // MoE totals among them (zeroed by a reset too)
    long long trace = 0;                  // 1: keep a record of every call (sim_comm_trace_read)
    std::vector<TraceSlot> trace_ring;    // the last kTraceCap calls
    unsigned long long trace_seq = 0;     // calls recorded so far
    unsigned long long trace_next = 0;    // seq of the oldest record not yet read
};

namespace {

thread_local std::string g_last_error;

coll_status_t fail(coll_status_t st, const std::string& msg) {
    g_last_error = msg;
    return st;
}

coll_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(COLL_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

size_t dtype_bytes(coll_dtype_t dt) { return dt == COLL_BF16 ? 2 : 4; }

bool valid_dtype(int dt) { return dt == COLL_INT32 || dt == COLL_FP32 || dt == COLL_BF16; }

coll_status_t check_reduce_args(coll_dtype_t dt, coll_op_t op) {
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if (op < COLL_SUM || op > COLL_AVG) return fail(COLL_ERR_INVALID_ARG, "unknown reduction op");
    if (dt == COLL_INT32 && op == COLL_AVG) return fail(COLL_ERR_UNSUPPORTED, "AVG is not defined for int32");
    return COLL_OK;
}

// Direct and ring exist for every collective; the butterfly algorithms for AllReduce only.
coll_status_t check_algo(coll_algo_t algo, bool allreduce = false, bool ll_ring = false) {
    if (algo == COLL_ALGO_DIRECT || algo == COLL_ALGO_RING) return COLL_OK;
    if (algo == COLL_ALGO_RING_LL && ll_ring) return COLL_OK;
    if (algo == COLL_ALGO_RD || algo == COLL_ALGO_HD || algo == COLL_ALGO_TREE || algo == COLL_ALGO_DBTREE ||
        algo == COLL_ALGO_RING_LL || algo == COLL_ALGO_RD_LL || algo == COLL_ALGO_TREE_LL ||
        algo == COLL_ALGO_DBTREE_LL) {
        if (allreduce) return COLL_OK;
        return fail(COLL_ERR_UNSUPPORTED,
                    "recursive doubling, halving-doubling, the trees and the LL ring exist for AllReduce only");
    }
    return fail(COLL_ERR_INVALID_ARG, "unknown algorithm");
}

// The sticky state: an abort requested on the host, or an asynchronous error already reported.
coll_status_t check_usable(sim_comm* c) {
    if (!c) return fail(COLL_ERR_INVALID_ARG, "null communicator");
    volatile uint32_t* hw = c->host_words;
    if (hw[1] != 0u) return fail(COLL_ERR_ABORTED, "communicator was aborted; call sim_comm_reset");
    if (hw[0] != 0u)
        return fail(coll_status_t(hw[0]), "communicator has an asynchronous error; call sim_comm_reset");
    return COLL_OK;
}

Ctl make_ctl(sim_comm* c) {
    Ctl ctl;
    ctl.status = &c->dstate->status;
    ctl.host_status = c->dev_words;
    ctl.abort_flag = c->dev_words + 1;
    ctl.abort_clock = &c->dstate->abort_clock;
    return ctl;
}

// ---- buffer validation -------------------------------------------------------------------------

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
    bool out;
    int rank;
};

bool overlap(const Range& a, const Range& b) { return a.lo < b.hi && b.lo < a.hi; }

// Allowed in-place pairs ([Primer] "In-place 不是“任意让输入输出指向同一地址”"): an output may
// coincide with or contain the SAME rank's input in the documented form only.
enum InPlaceRule { INPLACE_NONE, INPLACE_SAME, INPLACE_RS, INPLACE_AG };

bool allowed_pair(InPlaceRule rule, const Range& out, const Range& in, size_t shard_bytes) {
    if (out.rank != in.rank) return false;
    switch (rule) {
        case INPLACE_SAME: return out.lo == in.lo && out.hi == in.hi;
        case INPLACE_RS: return out.lo == in.lo + size_t(out.rank) * shard_bytes;  // recv = send + r*m
        case INPLACE_AG: return in.lo == out.lo + size_t(in.rank) * shard_bytes;   // send = recv + r*m
        default: return false;
    }
}

coll_status_t check_ranges(const std::vector<Range>& rs, InPlaceRule rule, size_t shard_bytes) {
    for (size_t i = 0; i < rs.size(); ++i) {
        for (size_t j = i + 1; j < rs.size(); ++j) {
            const Range& a = rs[i];
            const Range& b = rs[j];
            if (!a.out && !b.out) continue;  // inputs may share memory: they are only read
            if (a.lo == a.hi || b.lo == b.hi || !overlap(a, b)) continue;
            if (a.out && b.out) return fail(COLL_ERR_INVALID_ARG, "two output buffers overlap");
            const Range& o = a.out ? a : b;
            const Range& in = a.out ? b : a;
            if (!allowed_pair(rule, o, in, shard_bytes))
                return fail(COLL_ERR_INVALID_ARG, "an output overlaps an input outside the allowed in-place forms");
        }
    }
    return COLL_OK;
}

coll_status_t check_ptr(const void* p, size_t bytes, size_t elem, const char* what) {
    if (bytes == 0) return COLL_OK;
    if (!p) return fail(COLL_ERR_INVALID_ARG, std::string("null ") + what + " pointer");
    if (reinterpret_cast<uintptr_t>(p) % elem != 0)
        return fail(COLL_ERR_INVALID_ARG, std::string(what) + " pointer is not element-aligned");
    return COLL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest element count, capacity or row count x row length any entry point accepts. At 2^48
// elements every byte count and offset the host or a kernel forms (a count x an element of at most
// 8 bytes x 64 ranks, or a partial buffer of 4 bytes per element per rank) stays below 2^63, so no
// size computation can wrap around; a wrapped size would pass the pointer and scratch checks with a
// false small value. Checked before any multiplication.
constexpr size_t kMaxCount = size_t(1) << 48;

coll_status_t check_count(size_t n, const char* what) {
    if (n > kMaxCount)
        return fail(COLL_ERR_INVALID_ARG, std::string(what) + " exceeds 2^48 elements (" + std::to_string(n) + ")");
    return COLL_OK;
}

// A probe moves whole 16 KiB tiles, at most 2^48 bytes.
coll_status_t check_probe_bytes(size_t bytes) {
    if (bytes % (16 * 1024) != 0 || bytes > kMaxCount)
        return fail(COLL_ERR_INVALID_ARG, "probe bytes must be a multiple of 16 KiB, at most 2^48");
    return COLL_OK;
}

// rows x row length within kMaxCount, without forming the product first
coll_status_t check_rows(size_t rows, size_t row_elems, const char* what) {
    if (row_elems != 0 && rows > kMaxCount / row_elems)
        return fail(COLL_ERR_INVALID_ARG, std::string(what) + ": rows x hidden exceeds 2^48 elements");
    return COLL_OK;
}

void fill_ptrs(RankPtrs& rp, const coll_bufs_t& b, int p, bool use_send, bool use_recv) {
    std::memset(&rp, 0, sizeof(rp));
    for (int r = 0; r < p; ++r) {
        rp.send[r] = (use_send && b.send) ? b.send[r] : nullptr;
        rp.recv[r] = (use_recv && b.recv) ? b.recv[r] : nullptr;
    }
}

// ---- scratch -----------------------------------------------------------------------------------
// Scratch that a grown buffer replaces. A graph captured earlier keeps the old pointers in its
// kernel arguments and memset nodes, so once any call has been captured the old buffer stays
// allocated until the communicator is destroyed; before that it is freed at once (cudaFree
// synchronises the device, so no kernel still uses it).
void release_scratch(sim_comm* c, void* p) {
    if (!p) return;
    if (c->captured_any) c->retired.push_back(p);
    else cudaFree(p);
}

// Scratch grows with cudaMalloc/cudaFree, which a stream capture does not allow: under capture a
// call whose scratch is too small is refused (the same call made once before capturing sizes it).
coll_status_t grow_in_capture(const char* what) {
    return fail(COLL_ERR_UNSUPPORTED, std::string("the ") + what + " must grow, which a stream capture does not allow: "
                                      "make the same call once before capturing");
}

bool stream_capturing(cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone;
}

// Flags and LL slots tell this call's signals from older ones by the epoch or tag the host gives
// each call. A captured graph replays its call with the same epoch and tags, so under capture the
// region the call uses is cleared first, in stream order (a memset node of the graph).
coll_status_t clear_for_replay(sim_comm* c, void* p, size_t bytes, cudaStream_t s) {
    if (!c->capturing || bytes == 0) return COLL_OK;
    cudaError_t e = cudaMemsetAsync(p, 0, bytes, s);
    return e == cudaSuccess ? COLL_OK : cuda_fail(e, "cudaMemsetAsync(scratch cleared for graph replay)");
}


coll_status_t ensure_flags(sim_comm* c, size_t count) {
    if (count <= c->flags_cap) return COLL_OK;
    if (c->capturing) return grow_in_capture("ring flags");
    release_scratch(c, c->flags);
    c->flags = nullptr;
    c->flags_cap = 0;
    cudaError_t e = cudaMalloc(&c->flags, count * sizeof(unsigned long long));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(ring flags)");
    e = cudaMemset(c->flags, 0, count * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();  // zeroed before any stream's next kernel
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(ring flags)");
    c->flags_cap = count;
    return COLL_OK;
}

coll_status_t ensure_moe(sim_comm* c, size_t bytes) {
    if (bytes <= c->moe_cap) return COLL_OK;
    if (c->capturing) return grow_in_capture("MoE scratch");
    release_scratch(c, c->moe);
    c->moe = nullptr;
    c->moe_cap = 0;
    cudaError_t e = cudaMalloc(&c->moe, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(MoE scratch)");
    c->moe_cap = bytes;
    return COLL_OK;
}

// The fused dispatch sums its per-(rank, expert) totals into this array during counting, and the
// call's last CTA zeroes it again, so it is allocated zeroed and kept apart from the scratch whose
// layout changes with the call's shape.
coll_status_t ensure_moe_acc(sim_comm* c, size_t count) {
    if (count <= c->moe_acc_cap) return COLL_OK;
    if (c->capturing) return grow_in_capture("MoE totals");
    // a graph captured earlier keeps using the old array; a reset after a failed replay clears it too
    if (c->moe_acc && c->captured_any) c->retired_acc.push_back({c->moe_acc, c->moe_acc_cap});
    release_scratch(c, c->moe_acc);
    c->moe_acc = nullptr;
    c->moe_acc_cap = 0;
    cudaError_t e = cudaMalloc(&c->moe_acc, count * sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(MoE totals)");
    e = cudaMemset(c->moe_acc, 0, count * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();  // zeroed before any stream's next kernel
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(MoE totals)");
    c->moe_acc_cap = count;
    return COLL_OK;
}

coll_status_t ensure_stage(sim_comm* c, size_t bytes) {
    if (bytes <= c->stage_cap) return COLL_OK;
    if (c->capturing) return grow_in_capture("partial buffers");
    release_scratch(c, c->stage);
    c->stage = nullptr;
    c->stage_cap = 0;
    cudaError_t e = cudaMalloc(&c->stage, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(ring partial buffers)");
    c->stage_cap = bytes;
    return COLL_OK;
}

uint32_t next_epoch(sim_comm* c) {
    c->epoch += 1;
    if (c->epoch == 0) {  // wrapped: old flags could alias a future epoch, so clear them
        if (c->flags) cudaMemset(c->flags, 0, c->flags_cap * sizeof(unsigned long long));
        c->epoch = 1;
    }
    return c->epoch;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- launches ----------------------------------------------------------------------------------

coll_status_t run_direct_reduce(sim_comm* c, const coll_bufs_t& b, size_t n, coll_dtype_t dt, coll_op_t op,
                                int mode, int root, cudaStream_t s) {
    DirectReduceArgs a;
    fill_ptrs(a.ptrs, b, c->p, true, true);
    a.p = c->p;
    a.mode = mode;
    a.root = root;
    a.n = n;
    a.seg = (mode == MODE_REDUCE_SCATTER) ? n / size_t(c->p) : n;
    a.scale = (op == COLL_AVG) ? 1.0f / float(c->p) : 1.0f;
    a.ctl = make_ctl(c);
    const size_t d = dtype_bytes(dt);
    // The widest pack (32, then 16 bytes) every touched buffer is aligned to; ReduceScatter also
    // needs its owner segments to start on that boundary.
    auto all_aligned = [&](uintptr_t mask) {
        bool ok = true;
        for (int r = 0; r < c->p; ++r) ok = ok && (uintptr_t(a.ptrs.send[r]) & mask) == 0;
        if (mode == MODE_REDUCE) return ok && (uintptr_t(a.ptrs.recv[root]) & mask) == 0;
        for (int r = 0; r < c->p; ++r) ok = ok && (uintptr_t(a.ptrs.recv[r]) & mask) == 0;
        if (mode == MODE_REDUCE_SCATTER) ok = ok && ((a.seg * d) & mask) == 0;
        return ok;
    };
    a.vec = all_aligned(31) ? 2 : (all_aligned(15) ? 1 : 0);
    if (c->direct_pack == 16 && a.vec == 2) a.vec = 1;
    a.ctas_per_sm = int(c->direct_ctas_per_sm);
    a.l2_hint = c->l2_hint == 1 ? 1 : 0;  // the fused reduction hints its loads and stores together
    cudaError_t e = launch_direct_reduce(a, dt, op, c->num_sms, s);
    if (e != cudaSuccess) return cuda_fail(e, "direct reduction launch");
    c->launches += 1;
    return COLL_OK;
}

// p_override > 0: run the copy over that many segments' ranks instead of the communicator's p (a
// rank view's single-source copies).
coll_status_t run_copy(sim_comm* c, const coll_bufs_t& b, int kind, size_t blk_elems, coll_dtype_t dt, int root,
                       bool use_send_all, cudaStream_t s, const long long* counts = nullptr,
                       const long long* send_cap = nullptr, const long long* recv_cap = nullptr,
                       long long* recv_counts = nullptr, int p_override = 0, int only_dst = -1) {
    const int p = p_override > 0 ? p_override : c->p;
    CopyArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    if (!use_send_all)
        for (int r = 0; r < p; ++r)
            if (r != root) a.ptrs.send[r] = nullptr;
    a.p = p;
    a.kind = kind;
    a.root = root;
    a.elem_bytes = int(dtype_bytes(dt));
    a.blk_elems = blk_elems;
    a.counts = counts;
    a.recv_counts_out = recv_counts;
    for (int r = 0; r < p; ++r) {
        a.send_cap[r] = send_cap ? send_cap[r] : 0;
        a.recv_cap[r] = recv_cap ? recv_cap[r] : 0;
    }
    a.timeout_ns = uint64_t(c->timeout_ns);
    int variant = 0, order = 0;
    copy_defaults(kind, &variant, &order);
    if (c->copy_variant >= 0) variant = int(c->copy_variant);
    if (c->copy_order >= 0) order = int(c->copy_order);
    a.order = order;
    a.st = c->dstate;
    a.only_dst_plus1 = only_dst + 1;
    a.l2_hint = c->l2_hint >= 0 ? int(c->l2_hint) : copy_path_l2_hint(a, variant);
    a.ctl = make_ctl(c);
    cudaError_t e = launch_copy(a, c->num_sms, variant, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy engine launch");
    c->launches += 1;
    return COLL_OK;
}

struct RingPlan {
    int kind;
    size_t seg, chunk;
    uint32_t nch, nsteps, rps;
    bool needs_stage;
};

// One CTA task moves 128 KiB of the step's wire type (the partial type for reduce steps): a chunk
// is split into that many tasks so that several SMs carry one chunk through each step.
constexpr size_t kRingTaskBytes = 256 * 1024;  // bytes of the wire type one ring or tree task moves

// Task size of the ring and tree executors. Measured on B200 (p = 2..64): 256 KiB tasks are 2-6%
// faster than 128 KiB ones from 64 MiB of wire bytes per rank up, and 10-50% slower at 1-16 MiB,
// where the schedule needs more, shorter tasks per step to keep its pipeline full.
size_t default_task_bytes(size_t wire_bytes_per_rank) {
    return wire_bytes_per_rank >= (size_t(64) << 20) ? kRingTaskBytes : kRingTaskBytes / 2;
}

size_t task_bytes(const sim_comm* c, size_t wire_bytes_per_rank) {
    if (c->ring_task_bytes > 0) return size_t(c->ring_task_bytes);
    return default_task_bytes(wire_bytes_per_rank);
}

// CTA tasks of one ring chunk: a chunk spans at most `span` elements (a segment), and one task moves
// `task` bytes of the wire type (at least 16 elements).
void ring_tiles(size_t span, size_t wire, size_t task, size_t* tile, uint32_t* ntile) {
    *tile = std::min(span, std::max<size_t>(16, task / wire));
    *ntile = uint32_t((span + *tile - 1) / *tile);
}

coll_status_t run_ring(sim_comm* c, const coll_bufs_t& b, const RingPlan& pl, size_t n, coll_dtype_t dt,
                       coll_op_t op, int root, cudaStream_t s, const long long* counts = nullptr,
                       const long long* send_cap = nullptr, const long long* recv_cap = nullptr,
                       long long* recv_counts = nullptr) {
    const int p = c->p;
    const size_t d = dtype_bytes(dt);
    RingArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.p = p;
    a.kind = pl.kind;
    a.root = root;
    a.n = n;
    a.seg = pl.seg;
    a.chunk = pl.chunk;
    {
        const bool reduce_kind = (pl.kind == RING_ALLREDUCE || pl.kind == RING_REDUCE_SCATTER || pl.kind == RING_REDUCE);
        const size_t wire = reduce_kind ? 4 : d;
        // a chunk is at most a segment long (the All-to-Allv's block sizes are known on the device only)
        const size_t span = (pl.kind == RING_ALLTOALLV || pl.seg == 0) ? pl.chunk : std::min(pl.chunk, pl.seg);
        size_t per_rank = n * wire;  // the All-to-Allv's largest send buffer stands in for its message
        if (pl.kind == RING_ALLTOALLV && send_cap)
            for (int r = 0; r < p; ++r) per_rank = std::max(per_rank, size_t(std::max<long long>(send_cap[r], 0)) * d);
        ring_tiles(span, wire, task_bytes(c, per_rank), &a.tile, &a.ntile);
    }
    a.elem_bytes = int(d);
    a.nch = pl.nch;
    a.nsteps = pl.nsteps;
    a.ranks_per_step = pl.rps;
    a.scale = (op == COLL_AVG) ? 1.0f / float(p) : 1.0f;
    a.skip_rank = int(c->fault_skip_rank);
    a.timeout_ns = uint64_t(c->timeout_ns);
    a.counts = counts;
    a.recv_counts_out = recv_counts;
    for (int r = 0; r < p; ++r) {
        a.send_cap[r] = send_cap ? send_cap[r] : 0;
        a.recv_cap[r] = recv_cap ? recv_cap[r] : 0;
    }
    a.st = c->dstate;
    a.ctl = make_ctl(c);

    coll_status_t st;
    if (pl.kind != RING_ALLTOALL && pl.kind != RING_ALLTOALLV) {
        st = ensure_flags(c, size_t(pl.nsteps) * pl.rps * pl.nch);
        if (st != COLL_OK) return st;
    }
    if (pl.needs_stage) {
        a.stage_stride = round_up(n * 4, 256);
        st = ensure_stage(c, a.stage_stride * size_t(p));
        if (st != COLL_OK) return st;
        a.stage = c->stage;
    }
    a.flags = c->flags;
    a.epoch = next_epoch(c);
    if (pl.kind != RING_ALLTOALL && pl.kind != RING_ALLTOALLV) {
        st = clear_for_replay(c, c->flags, size_t(pl.nsteps) * pl.rps * pl.nch * sizeof(unsigned long long), s);
        if (st != COLL_OK) return st;
    }

    // 16-byte hops need every segment and chunk start 16-byte aligned in the element and partial
    // buffers, and 16-byte aligned bases.
    const bool chain = (pl.kind == RING_REDUCE || pl.kind == RING_BCAST);  // chunks of [0, n), no segments
    bool vec = (chain || ((pl.seg * d) % 16 == 0 && (pl.seg * 4) % 16 == 0)) && (pl.chunk * d) % 16 == 0;
    for (int r = 0; r < p; ++r)
        vec = vec && (!a.ptrs.send[r] || aligned16(a.ptrs.send[r])) && (!a.ptrs.recv[r] || aligned16(a.ptrs.recv[r]));
    a.vec = vec ? 1 : 0;

    int ctas = int(c->ring_ctas > 0 ? c->ring_ctas : c->ring_ctas_max);
    if (pl.kind != RING_ALLTOALLV) {
        const size_t tasks = size_t(pl.nsteps) * pl.rps * pl.nch * a.ntile;
        if (tasks < size_t(ctas)) ctas = int(std::max<size_t>(tasks, 1));
    }
    cudaError_t e = launch_ring(a, dt, op, ctas, s);
    if (e != cudaSuccess) return cuda_fail(e, "ring executor launch");
    c->launches += 1;
    return COLL_OK;
}

// The LL protocol's receive slots (flags inside the data): grown on demand, never cleared between
// calls because tags never repeat while old words may sit in them.
constexpr size_t kLLMaxBytes = size_t(256) << 20;

coll_status_t ensure_ll_slots(sim_comm* c, size_t bytes) {
    if (bytes > kLLMaxBytes)
        return fail(COLL_ERR_UNSUPPORTED, "the LL protocol is for small messages: its receive slots must stay "
                                          "within 256 MiB (use COLL_ALGO_RING or COLL_ALGO_RD)");
    if (bytes <= c->ll_cap) return COLL_OK;
    if (c->capturing) return grow_in_capture("LL slots");
    release_scratch(c, c->ll);
    c->ll = nullptr;
    c->ll_cap = 0;
    cudaError_t e = cudaMalloc(&c->ll, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(LL slots)");
    e = cudaMemset(c->ll, 0, bytes);  // tag 0 is never a live tag
    if (e == cudaSuccess) e = cudaDeviceSynchronize();  // zeroed before any stream's next kernel
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(LL slots)");
    c->ll_cap = bytes;
    return COLL_OK;
}

// This call's tag of slot 0 (slot q carries tag + q, q < 128). Before e * 128 + 127 would leave 32
// bits the counter starts again and the slots are cleared, in stream order.
coll_status_t next_ll_tag(sim_comm* c, cudaStream_t s, uint32_t* tag) {
    c->ll_epoch += 1;
    if (c->ll_epoch >= (1u << 25)) {
        cudaError_t e = cudaMemsetAsync(c->ll, 0, c->ll_cap, s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(LL slots)");
        c->ll_epoch = 1;
    }
    *tag = c->ll_epoch * 128u + 1u;
    return COLL_OK;
}

coll_status_t launch_ll(sim_comm* c, LLArgs& a, coll_dtype_t dt, coll_op_t op, cudaStream_t s) {
    a.ll = c->ll;
    a.scale = (op == COLL_AVG) ? 1.0f / float(a.p) : 1.0f;
    a.skip_rank = int(c->fault_skip_rank);
    a.timeout_ns = uint64_t(c->timeout_ns);
    a.ctl = make_ctl(c);
    cudaError_t e = launch_ring_ll(a, dt, op, s);
    if (e != cudaSuccess) return cuda_fail(e, "LL launch");
    c->launches += 1;
    return COLL_OK;
}

int ll_ctas_cap(sim_comm* c) {
    if (c->ll_ctas_max == 0) c->ll_ctas_max = ring_ll_max_ctas(c->num_sms);
    return c->ll_ctas_max;
}

// Ring AllReduce / ReduceScatter / AllGather on the low-latency protocol, for small messages. n is
// the per-rank full buffer (the AllReduce buffer, the ReduceScatter input, the AllGather output).
coll_status_t run_ring_ll(sim_comm* c, const coll_bufs_t& b, size_t n, coll_dtype_t dt, coll_op_t op, cudaStream_t s,
                          int kind = LL_RING) {
    const int p = c->p;
    LLArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.kind = kind;
    a.p = p;
    a.n = n;
    a.seg = (n + size_t(p) - 1) / size_t(p);
    a.nslots = uint32_t(kind == LL_RING ? 2 * p - 3 : p - 2);  // one per step that crosses a hop
    coll_status_t st = ensure_ll_slots(c, size_t(p) * a.nslots * a.seg * sizeof(unsigned long long));
    if (st != COLL_OK) return st;
    if ((st = next_ll_tag(c, s, &a.tag)) != COLL_OK) return st;
    if ((st = clear_for_replay(c, c->ll, size_t(p) * a.nslots * a.seg * sizeof(unsigned long long), s)) != COLL_OK)
        return st;
    // CTAs per rank: about 4 elements per thread, all CTAs resident at once (cooperative launch)
    const int g_cap = ll_ctas_cap(c) / p;
    if (g_cap < 1) return fail(COLL_ERR_UNSUPPORTED, "too many ranks for one resident LL grid");
    a.G = int(std::max<size_t>(1, std::min<size_t>((a.seg + 1023) / 1024, size_t(g_cap))));
    return launch_ll(c, a, dt, op, s);
}

// Single or double binary tree AllReduce on the low-latency protocol: three slots per rank (left
// child, right child, parent), any p. The double tree sends elements [ceil(n/2), n) over the mirror
// tree, in CTAs of their own.
coll_status_t run_tree_ll(sim_comm* c, const coll_bufs_t& b, size_t n, coll_dtype_t dt, coll_op_t op, bool dbl,
                          cudaStream_t s) {
    const int p = c->p;
    LLArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.kind = LL_TREE;
    a.p = p;
    a.n = n;
    a.seg = dbl ? (n + 1) / 2 : n;  // elements of tree A
    a.nslots = 3;
    coll_status_t st = ensure_ll_slots(c, size_t(p) * a.nslots * n * sizeof(unsigned long long));
    if (st != COLL_OK) return st;
    if ((st = next_ll_tag(c, s, &a.tag)) != COLL_OK) return st;
    if ((st = clear_for_replay(c, c->ll, size_t(p) * a.nslots * n * sizeof(unsigned long long), s)) != COLL_OK)
        return st;
    // CTAs per rank and tree: about 4 elements per thread, all CTAs resident at once
    const int g_cap = ll_ctas_cap(c) / p;
    if (g_cap < (dbl ? 2 : 1)) return fail(COLL_ERR_UNSUPPORTED, "too many ranks for one resident LL grid");
    const size_t nb = n - a.seg;
    const int g_tree = dbl ? g_cap / 2 : g_cap;
    a.GA = int(std::max<size_t>(1, std::min<size_t>((a.seg + 1023) / 1024, size_t(g_tree))));
    const int gb = nb ? int(std::max<size_t>(1, std::min<size_t>((nb + 1023) / 1024, size_t(g_tree)))) : 0;
    a.G = a.GA + gb;
    return launch_ll(c, a, dt, op, s);
}

// Recursive-doubling AllReduce on the low-latency protocol: every rank's whole vector in registers
// of one resident grid, at most 8 elements per thread.
coll_status_t run_rd_ll(sim_comm* c, const coll_bufs_t& b, size_t n, coll_dtype_t dt, coll_op_t op, cudaStream_t s) {
    const int p = c->p;
    if (p & (p - 1)) return fail(COLL_ERR_UNSUPPORTED, "recursive doubling needs p a power of two");
    int L = 0;
    while ((1 << L) < p) ++L;
    LLArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.kind = LL_RD;
    a.p = p;
    a.n = n;
    a.seg = n;
    a.nslots = uint32_t(L);
    const int g_cap = ll_ctas_cap(c) / p;
    if (g_cap < 1) return fail(COLL_ERR_UNSUPPORTED, "too many ranks for one resident LL grid");
    const size_t per_thread = (n + size_t(g_cap) * 256 - 1) / (size_t(g_cap) * 256);
    if (per_thread > 8)
        return fail(COLL_ERR_UNSUPPORTED, "the LL recursive doubling holds at most 8 elements per thread of one "
                                          "resident grid (use COLL_ALGO_RD for larger messages)");
    a.ept = per_thread <= 1 ? 1 : per_thread <= 2 ? 2 : per_thread <= 4 ? 4 : 8;
    // CTAs per rank: the fewest that keep ept elements per thread
    a.G = int(std::max<size_t>(1, (n + size_t(a.ept) * 256 - 1) / (size_t(a.ept) * 256)));
    coll_status_t st = ensure_ll_slots(c, size_t(p) * a.nslots * n * sizeof(unsigned long long));
    if (st != COLL_OK) return st;
    if ((st = next_ll_tag(c, s, &a.tag)) != COLL_OK) return st;
    if ((st = clear_for_replay(c, c->ll, size_t(p) * a.nslots * n * sizeof(unsigned long long), s)) != COLL_OK)
        return st;
    return launch_ll(c, a, dt, op, s);
}

// Single / double binary tree AllReduce on the tree executor.
coll_status_t run_tree(sim_comm* c, const coll_bufs_t& b, size_t n, coll_dtype_t dt, coll_op_t op, bool dbl,
                       cudaStream_t s) {
    const int p = c->p;
    const size_t d = dtype_bytes(dt);
    TreeArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.p = p;
    a.ntrees = dbl ? 2 : 1;
    a.n = n;
    a.half = dbl ? (n + 1) / 2 : n;
    a.chunk = size_t(c->chunk_bytes) / 4;  // chunk bytes count the fp32/int32 partials, as on the ring
    a.tile = std::min(a.chunk, task_bytes(c, n * 4) / 4);
    a.ntile = uint32_t((a.chunk + a.tile - 1) / a.tile);
    const size_t len[2] = {a.half, n - a.half};
    for (int t = 0; t < a.ntrees; ++t) a.nch[t] = uint32_t((len[t] + a.chunk - 1) / a.chunk);
    a.nchmax = std::max(a.nch[0], a.nch[1]);
    // a short range is one chunk cut into about 4 tasks (parallelism within each level) of whole
    // 64-element packs, at least 1024 elements each, so no task is empty
    if (a.nchmax == 1) {
        const size_t longest = std::max(len[0], len[1]);
        const size_t quarter = round_up(std::max<size_t>((longest + 3) / 4, 1024), 64);
        a.tile = std::min(a.tile, quarter);
        a.ntile = uint32_t((longest + a.tile - 1) / a.tile);
        a.chunk = size_t(a.ntile) * a.tile;
    }
    // levels: internal positions (2m+1 < p) reduce, deepest level first; then every non-root
    // position copies its parent's result, root side first
    auto level_of = [](int m) { int L = 0; while ((2 << L) <= m + 1) ++L; return L; };
    const int internal_last = p / 2 - 1, depth = level_of(p - 1);
    const int reduce_levels = level_of(internal_last) + 1;
    uint32_t g = 0;
    for (int L = reduce_levels - 1; L >= 0; --L, ++g) {
        a.step_kind[g] = 0;
        a.step_first[g] = uint32_t((1 << L) - 1);
        a.step_count[g] = uint32_t(std::min((2 << L) - 1, internal_last + 1) - ((1 << L) - 1));
    }
    for (int L = 1; L <= depth; ++L, ++g) {
        a.step_kind[g] = 1;
        a.step_first[g] = uint32_t((1 << L) - 1);
        a.step_count[g] = uint32_t(std::min((2 << L) - 1, p) - ((1 << L) - 1));
    }
    a.nsteps = g;
    a.start[0] = 0;
    for (uint32_t k = 0; k < a.nsteps; ++k)
        a.start[k + 1] = a.start[k] + (a.nch[0] + (a.ntrees == 2 ? a.nch[1] : 0)) * a.step_count[k] * a.ntile;
    a.scale = (op == COLL_AVG) ? 1.0f / float(p) : 1.0f;
    a.skip_rank = int(c->fault_skip_rank);
    a.timeout_ns = uint64_t(c->timeout_ns);
    a.st = c->dstate;
    a.ctl = make_ctl(c);
    coll_status_t st = ensure_flags(c, size_t(4) * p * a.nchmax);
    if (st != COLL_OK) return st;
    a.flags = c->flags;
    a.epoch = next_epoch(c);
    if ((st = clear_for_replay(c, c->flags, size_t(4) * p * a.nchmax * sizeof(unsigned long long), s)) != COLL_OK)
        return st;
    a.stage_stride = round_up(n * 4, 256);
    if ((st = ensure_stage(c, a.stage_stride * size_t(p))) != COLL_OK) return st;
    a.stage = c->stage;
    // 16-byte packs need every range start (chunk and tile starts, and the second tree's start) on a
    // 16-byte boundary of the element and of the partial buffers
    bool vec = (a.tile * d) % 16 == 0 && (a.tile * 4) % 16 == 0 && (a.chunk * d) % 16 == 0 && (a.chunk * 4) % 16 == 0;
    if (a.ntrees == 2) vec = vec && (a.half * d) % 16 == 0 && (a.half * 4) % 16 == 0;
    for (int r = 0; r < p; ++r) vec = vec && aligned16(a.ptrs.send[r]) && aligned16(a.ptrs.recv[r]);
    a.vec = vec ? 1 : 0;
    int ctas = c->ring_ctas > 0 ? int(c->ring_ctas) : c->ring_ctas_max;
    if (a.start[a.nsteps] < uint32_t(ctas)) ctas = int(std::max<uint32_t>(a.start[a.nsteps], 1));
    cudaError_t e = launch_tree(a, dt, op, ctas, s);
    if (e != cudaSuccess) return cuda_fail(e, "tree executor launch");
    c->launches += 1;
    return COLL_OK;
}

// Recursive doubling / halving-doubling AllReduce on the butterfly executor.
coll_status_t run_butterfly(sim_comm* c, const coll_bufs_t& b, size_t n, coll_dtype_t dt, coll_op_t op, int kind,
                            cudaStream_t s) {
    const int p = c->p;
    if (p & (p - 1)) return fail(COLL_ERR_UNSUPPORTED, "recursive doubling / halving-doubling need p a power of two");
    int L = 0;
    while ((1 << L) < p) ++L;
    const size_t d = dtype_bytes(dt);
    ButterflyArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.p = p;
    a.kind = kind;
    a.log2p = L;
    a.n = n;
    a.seg = (n + size_t(p) - 1) / size_t(p);
    a.tile = 32768;  // 128 KiB of fp32/int32 partials per CTA task
    a.nsteps = uint32_t(kind == BFLY_RD ? L : 2 * L);
    a.start[0] = 0;
    for (uint32_t g = 0; g < a.nsteps; ++g) {
        size_t elems;  // the most elements one rank handles at step g
        if (kind == BFLY_RD) elems = n;
        else if (int(g) < L) elems = size_t(p >> (g + 1)) * a.seg;    // the kept half of a block group
        else elems = (size_t(1) << (int(g) - L)) * a.seg;             // the partner's group of blocks
        elems = std::min(elems, n);
        a.ntile[g] = uint32_t(std::max<size_t>(1, (elems + a.tile - 1) / a.tile));
        a.start[g + 1] = a.start[g] + uint32_t(p) * a.ntile[g];
    }
    a.scale = (op == COLL_AVG) ? 1.0f / float(p) : 1.0f;
    a.skip_rank = int(c->fault_skip_rank);
    a.timeout_ns = uint64_t(c->timeout_ns);
    a.st = c->dstate;
    a.ctl = make_ctl(c);
    a.stage_stride = round_up(n * 4, 256);
    const size_t nbuf = (kind == BFLY_RD) ? 2 * size_t(p) : size_t(p);
    if (L > 1 || kind == BFLY_HD) {
        coll_status_t st = ensure_stage(c, a.stage_stride * nbuf);
        if (st != COLL_OK) return st;
        a.stage = c->stage;
    }
    bool vec = (kind == BFLY_RD) || ((a.seg * d) % 16 == 0 && (a.seg * 4) % 16 == 0);
    for (int r = 0; r < p; ++r) vec = vec && aligned16(a.ptrs.send[r]) && aligned16(a.ptrs.recv[r]);
    a.vec = vec ? 1 : 0;
    int ctas = c->ring_ctas > 0 ? int(c->ring_ctas) : c->ring_ctas_max;
    if (a.start[a.nsteps] < uint32_t(ctas)) ctas = int(std::max<uint32_t>(a.start[a.nsteps], 1));
    cudaError_t e = launch_butterfly(a, dt, op, ctas, s);
    if (e != cudaSuccess) return cuda_fail(e, "butterfly executor launch");
    c->launches += 1;
    return COLL_OK;
}

uint32_t chunks_of(size_t seg, size_t chunk) { return uint32_t(std::max<size_t>(1, (seg + chunk - 1) / chunk)); }

constexpr const char* kOptionKeys[] = {"chunk_bytes", "ring_ctas", "ring_task_bytes", "timeout_ns",
                                       "fault_skip_rank", "copy_variant", "copy_order", "direct_pack",
                                       "direct_ctas_per_sm", "l2_hint", "moe_tma", "moe_fused", "trace"};

coll_status_t set_option_impl(sim_comm* c, const char* key, long long value) {
    std::string k(key);
    if (k == "chunk_bytes") {
        if (value < 256 || value % 256 != 0 || value > (1LL << 30))
            return fail(COLL_ERR_INVALID_ARG, "chunk_bytes must be a multiple of 256 in [256, 2^30]");
        c->chunk_bytes = value;
    } else if (k == "ring_ctas") {
        if (value < 0 || value > 65535) return fail(COLL_ERR_INVALID_ARG, "ring_ctas out of range");
        c->ring_ctas = value;
    } else if (k == "timeout_ns") {
        if (value < 1000) return fail(COLL_ERR_INVALID_ARG, "timeout_ns must be at least 1000");
        c->timeout_ns = value;
    } else if (k == "fault_skip_rank") {
        if (value < -1 || value >= c->p) return fail(COLL_ERR_INVALID_ARG, "fault_skip_rank out of range");
        c->fault_skip_rank = value;
    } else if (k == "copy_variant") {
        if (value < -1 || value >= copy_num_variants()) return fail(COLL_ERR_INVALID_ARG, "copy_variant out of range");
        c->copy_variant = value;
    } else if (k == "copy_order") {
        if (value < -1 || value > 1) return fail(COLL_ERR_INVALID_ARG, "copy_order must be -1, 0 or 1");
        c->copy_order = value;
    } else if (k == "l2_hint") {
        if (value < -1 || value > 2) return fail(COLL_ERR_INVALID_ARG, "l2_hint must be -1, 0, 1 or 2");
        c->l2_hint = value;
    } else if (k == "direct_pack") {
        if (value != 0 && value != 16 && value != 32) return fail(COLL_ERR_INVALID_ARG, "direct_pack must be 0, 16 or 32");
        c->direct_pack = value;
    } else if (k == "direct_ctas_per_sm") {
        if (value < 0 || value > 32) return fail(COLL_ERR_INVALID_ARG, "direct_ctas_per_sm must be in [0, 32]");
        c->direct_ctas_per_sm = value;
    } else if (k == "ring_task_bytes") {
        if (value != 0 && (value < 4096 || value > (64 << 20) || value % 256 != 0))
            return fail(COLL_ERR_INVALID_ARG, "ring_task_bytes must be 0 or a multiple of 256 in [4 KiB, 64 MiB]");
        c->ring_task_bytes = value;
    } else if (k == "moe_tma") {
        if (value != 0 && value != 1) return fail(COLL_ERR_INVALID_ARG, "moe_tma must be 0 or 1");
        c->moe_tma = value;
    } else if (k == "moe_fused") {
        if (value != 0 && value != 1) return fail(COLL_ERR_INVALID_ARG, "moe_fused must be 0 or 1");
        c->moe_fused = value;
    } else if (k == "trace") {
        if (value != 0 && value != 1) return fail(COLL_ERR_INVALID_ARG, "trace must be 0 or 1");
        c->trace = value;
    } else {
        return fail(COLL_ERR_INVALID_ARG, "unknown option " + k);
    }
    return COLL_OK;
}

// Brackets one entry-point call: an NVTX range (seen by a profiler that collects NVTX; a no-op
// otherwise), notes whether the call's stream is being captured into a graph, and, while the
// communicator's "trace" option is on, records the call with CUDA events around its kernels (not on
// a stream that is being captured).
struct TraceScope {
    sim_comm* c = nullptr;
    TraceSlot* slot = nullptr;
    cudaStream_t s = nullptr;
    unsigned long long launches0 = 0;

    TraceScope(sim_comm* comm, const char* coll, size_t n, int dtype, int op, int root, int algo,
               coll_stream_t stream) {
        nvtxRangePushA(coll);
        if (!comm) return;
        comm->capturing = stream_capturing(static_cast<cudaStream_t>(stream));
        if (comm->capturing) comm->captured_any = true;
        if (!comm->trace) return;
        c = comm;
        s = static_cast<cudaStream_t>(stream);
        if (c->trace_ring.size() < kTraceCap) c->trace_ring.resize(kTraceCap);
        slot = &c->trace_ring[c->trace_seq % kTraceCap];
        slot->rec = sim_comm_trace_record_t{};
        slot->rec.seq = c->trace_seq;
        slot->rec.coll = coll;
        slot->rec.p = c->p;
        slot->rec.n = n;
        slot->rec.dtype = dtype;
        slot->rec.op = op;
        slot->rec.root = root;
        slot->rec.algo = algo;
        slot->rec.device_ms = -1.0f;
        slot->timed = !c->capturing;
        if (slot->timed && !slot->ev0)
            slot->timed = cudaEventCreate(&slot->ev0) == cudaSuccess && cudaEventCreate(&slot->ev1) == cudaSuccess;
        if (slot->timed) slot->timed = cudaEventRecord(slot->ev0, s) == cudaSuccess;
        launches0 = c->launches;
    }

    coll_status_t done(coll_status_t st) {
        if (slot) {
            slot->rec.status = int(st);
            slot->rec.launches = unsigned(c->launches - launches0);
            if (slot->timed) slot->timed = cudaEventRecord(slot->ev1, s) == cudaSuccess;
            c->trace_seq += 1;
            if (c->trace_seq - c->trace_next > kTraceCap) c->trace_next = c->trace_seq - kTraceCap;
        }
        nvtxRangePop();
        return st;
    }
};

// ---- rank views: one rank of a communicator whose ranks are separate processes -------------------
// The process of rank r holds a rank view (sim_comm_create_rank). bufs.send[q] is rank q's input as
// this process maps it (its own buffer for q = r, a mapping from sim_ipc_open of rank q's buffer
// otherwise) and bufs.recv[r] this rank's output; the other recv entries are ignored. A call
// computes rank r's output only, reading every rank's input where it lies (a pull), with the same
// kernels, fold order and rounding as the whole communicator's direct path, so rank r's output
// equals that path's output for rank r bit for bit ([Atlas] §3.3: the P2P transport reads a peer's
// buffer directly).

enum RankColl { RK_ALLREDUCE, RK_REDUCE, RK_BCAST, RK_REDUCE_SCATTER, RK_ALLGATHER, RK_ALLTOALL, RK_SCATTER, RK_GATHER };

// Checks the inputs this rank reads (every rank's, or only src_rank's) and its own output.
coll_status_t rank_check(sim_comm* c, const coll_bufs_t& b, size_t in_bytes, size_t out_bytes, size_t d,
                         int src_rank, InPlaceRule rule, size_t shard_bytes) {
    coll_status_t st;
    std::vector<Range> rs;
    for (int q = 0; q < c->p; ++q) {
        if (src_rank >= 0 && q != src_rank) continue;
        if ((st = check_ptr(b.send[q], in_bytes, d, "send")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[q]), uintptr_t(b.send[q]) + in_bytes, false, q});
    }
    if ((st = check_ptr(b.recv[c->rank], out_bytes, d, "recv")) != COLL_OK) return st;
    rs.push_back({uintptr_t(b.recv[c->rank]), uintptr_t(b.recv[c->rank]) + out_bytes, true, c->rank});
    return check_ranges(rs, rule, shard_bytes);
}

coll_status_t rank_collective(sim_comm* c, RankColl coll, const coll_bufs_t& b, size_t n, coll_dtype_t dt,
                              coll_op_t op, int root, coll_algo_t algo, cudaStream_t s) {
    if (algo != COLL_ALGO_DIRECT)
        return fail(COLL_ERR_UNSUPPORTED, "a rank view runs the direct path only (the ring, tree and LL schedules "
                                          "wait on other ranks inside their kernels)");
    const int p = c->p, r = c->rank;
    if ((coll == RK_REDUCE || coll == RK_GATHER) && r != root) return COLL_OK;  // only the root has an output
    const size_t d = dtype_bytes(dt), m = n / size_t(p);
    std::vector<const void*> send(p, nullptr);
    std::vector<void*> recv(p, nullptr);
    recv[r] = b.recv[r];
    coll_status_t st;
    switch (coll) {
        case RK_ALLREDUCE:
        case RK_REDUCE:
            if ((st = rank_check(c, b, n * d, n * d, d, -1, INPLACE_NONE, 0)) != COLL_OK) return st;
            for (int q = 0; q < p; ++q) send[q] = b.send[q];
            return run_direct_reduce(c, coll_bufs_t{send.data(), recv.data()}, n, dt, op, MODE_REDUCE, r, s);
        case RK_REDUCE_SCATTER:  // this rank's block of every input, reduced
            if ((st = rank_check(c, b, n * d, m * d, d, -1, INPLACE_NONE, 0)) != COLL_OK) return st;
            for (int q = 0; q < p; ++q) send[q] = static_cast<const char*>(b.send[q]) + size_t(r) * m * d;
            return run_direct_reduce(c, coll_bufs_t{send.data(), recv.data()}, m, dt, op, MODE_REDUCE, r, s);
        case RK_ALLGATHER:  // every rank's shard, gathered into this rank's output
        case RK_GATHER:
            if ((st = rank_check(c, b, m * d, n * d, d, -1, INPLACE_NONE, 0)) != COLL_OK) return st;
            for (int q = 0; q < p; ++q) send[q] = b.send[q];
            return run_copy(c, coll_bufs_t{send.data(), recv.data()}, COPY_GATHER, m, dt, r, true, s);
        case RK_ALLTOALL:  // block r of every rank's input
            if ((st = rank_check(c, b, n * d, n * d, d, -1, INPLACE_NONE, 0)) != COLL_OK) return st;
            for (int q = 0; q < p; ++q) send[q] = static_cast<const char*>(b.send[q]) + size_t(r) * m * d;
            return run_copy(c, coll_bufs_t{send.data(), recv.data()}, COPY_GATHER, m, dt, r, true, s);
        case RK_BCAST:  // the root's input copied to this rank's output (the root's own in place: nothing)
        case RK_SCATTER: {  // block r of the root's input
            const bool bc = coll == RK_BCAST;
            if ((st = rank_check(c, b, n * d, (bc ? n : m) * d, d, root, bc ? INPLACE_SAME : INPLACE_RS, m * d)) !=
                COLL_OK)
                return st;
            const void* src[1] = {static_cast<const char*>(b.send[root]) + (bc ? 0 : size_t(r) * m * d)};
            void* dst[1] = {b.recv[r]};
            return run_copy(c, coll_bufs_t{src, dst}, COPY_GATHER, bc ? n : m, dt, 0, true, s, nullptr, nullptr,
                            nullptr, nullptr, 1);
        }
    }
    return fail(COLL_ERR_INTERNAL, "unknown rank-view collective");
}

}  // namespace

// =================================================================================================
extern "C" {

const char* sim_comm_last_error(void) { return g_last_error.c_str(); }

const char* coll_status_string(coll_status_t s) {
    switch (s) {
        case COLL_OK: return "COLL_OK";
        case COLL_ERR_INVALID_ARG: return "COLL_ERR_INVALID_ARG";
        case COLL_ERR_UNSUPPORTED: return "COLL_ERR_UNSUPPORTED";
        case COLL_ERR_CUDA: return "COLL_ERR_CUDA";
        case COLL_ERR_TIMEOUT: return "COLL_ERR_TIMEOUT";
        case COLL_ERR_ABORTED: return "COLL_ERR_ABORTED";
        case COLL_ERR_OVERFLOW: return "COLL_ERR_OVERFLOW";
        case COLL_ERR_INTERNAL: return "COLL_ERR_INTERNAL";
        default: return "COLL_ERR_UNKNOWN";
    }
}

sim_comm_t sim_comm_create(int p) {
    if (p < 1 || p > SIM_COMM_MAX_RANKS) {
        fail(COLL_ERR_INVALID_ARG, "p must be in [1, 64]");
        return nullptr;
    }
    sim_comm* c = new sim_comm();
    c->p = p;
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
    if (e == cudaSuccess) e = cudaMalloc(&c->dstate, sizeof(DevState));
    if (e == cudaSuccess) e = cudaMemset(c->dstate, 0, sizeof(DevState));
    if (e == cudaSuccess) e = cudaHostAlloc(&c->host_words, 64, cudaHostAllocMapped);
    if (e == cudaSuccess) {
        std::memset(c->host_words, 0, 64);
        e = cudaHostGetDevicePointer(&c->dev_words, c->host_words, 0);
    }
    if (e != cudaSuccess) {
        cuda_fail(e, "sim_comm_create");
        if (c->dstate) cudaFree(c->dstate);
        if (c->host_words) cudaFreeHost(c->host_words);
        delete c;
        return nullptr;
    }
    c->ring_ctas_max = ring_max_ctas(c->num_sms);
    // Options from the environment (SIMCOMM_<KEY>); a value the option rejects leaves the default.
    for (const char* key : kOptionKeys) {
        std::string env = "SIMCOMM_";
        for (const char* q = key; *q; ++q) env += char(std::toupper(static_cast<unsigned char>(*q)));
        const char* v = std::getenv(env.c_str());
        if (!v || !*v) continue;
        char* end = nullptr;
        const long long x = std::strtoll(v, &end, 0);
        if (end && *end == 0) set_option_impl(c, key, x);
    }
    g_last_error.clear();
    return c;
}

sim_comm_t sim_comm_create_rank(int p, int rank) {
    if (p < 1 || p > SIM_COMM_MAX_RANKS || rank < 0 || rank >= p) {
        fail(COLL_ERR_INVALID_ARG, "p must be in [1, 64] and rank in [0, p)");
        return nullptr;
    }
    sim_comm_t c = sim_comm_create(p);
    if (c) c->rank = rank;
    return c;
}

int sim_comm_rank(sim_comm_t c) { return c ? c->rank : -2; }

coll_status_t sim_ipc_alloc(size_t bytes, void** dev_ptr, sim_ipc_handle_t* handle) {
    static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(sim_ipc_handle_t), "handle sizes differ");
    if (!dev_ptr || !handle || bytes == 0) return fail(COLL_ERR_INVALID_ARG, "null argument or zero bytes");
    if (bytes > kMaxCount) return fail(COLL_ERR_INVALID_ARG, "bytes exceed 2^48");
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(shared buffer)");
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, p);
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e, "cudaIpcGetMemHandle");
    }
    std::memcpy(handle, &h, sizeof(h));
    *dev_ptr = p;
    return COLL_OK;
}

coll_status_t sim_ipc_free(void* dev_ptr) {
    if (!dev_ptr) return COLL_OK;
    cudaError_t e = cudaFree(dev_ptr);
    return e == cudaSuccess ? COLL_OK : cuda_fail(e, "cudaFree(shared buffer)");
}

coll_status_t sim_ipc_open(const sim_ipc_handle_t* handle, void** peer_ptr) {
    if (!handle || !peer_ptr) return fail(COLL_ERR_INVALID_ARG, "null argument");
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    cudaError_t e = cudaIpcOpenMemHandle(peer_ptr, h, cudaIpcMemLazyEnablePeerAccess);
    return e == cudaSuccess ? COLL_OK : cuda_fail(e, "cudaIpcOpenMemHandle");
}

coll_status_t sim_ipc_close(void* peer_ptr) {
    if (!peer_ptr) return COLL_OK;
    cudaError_t e = cudaIpcCloseMemHandle(peer_ptr);
    return e == cudaSuccess ? COLL_OK : cuda_fail(e, "cudaIpcCloseMemHandle");
}

coll_status_t sim_comm_destroy(sim_comm_t c) {
    if (!c) return COLL_OK;
    cudaDeviceSynchronize();
    if (c->flags) cudaFree(c->flags);
    if (c->stage) cudaFree(c->stage);
    if (c->moe) cudaFree(c->moe);
    if (c->moe_acc) cudaFree(c->moe_acc);
    if (c->ll) cudaFree(c->ll);
    if (c->dstate) cudaFree(c->dstate);
    if (c->host_words) cudaFreeHost(c->host_words);
    for (void* q : c->retired) cudaFree(q);
    for (TraceSlot& t : c->trace_ring) {
        if (t.ev0) cudaEventDestroy(t.ev0);
        if (t.ev1) cudaEventDestroy(t.ev1);
    }
    delete c;
    return COLL_OK;
}

coll_status_t sim_comm_trace_read(sim_comm_t c, sim_comm_trace_record_t* out, int cap, int* count) {
    if (!c || !count || cap < 0 || (cap > 0 && !out)) return fail(COLL_ERR_INVALID_ARG, "null argument or negative cap");
    int got = 0;
    while (got < cap && c->trace_next < c->trace_seq) {
        TraceSlot& t = c->trace_ring[c->trace_next % kTraceCap];
        out[got] = t.rec;
        if (t.timed && t.rec.launches > 0) {
            float ms = -1.0f;
            if (cudaEventSynchronize(t.ev1) == cudaSuccess && cudaEventElapsedTime(&ms, t.ev0, t.ev1) == cudaSuccess)
                out[got].device_ms = ms;
        }
        ++got;
        ++c->trace_next;
    }
    *count = got;
    return COLL_OK;
}

int sim_comm_size(sim_comm_t c) { return c ? c->p : -1; }

coll_status_t sim_comm_set_option(sim_comm_t c, const char* key, long long value) {
    if (!c || !key) return fail(COLL_ERR_INVALID_ARG, "null communicator or key");
    return set_option_impl(c, key, value);
}

coll_status_t sim_comm_get_option(sim_comm_t c, const char* key, long long* value) {
    if (!c || !key || !value) return fail(COLL_ERR_INVALID_ARG, "null argument");
    std::string k(key);
    if (k == "chunk_bytes") *value = c->chunk_bytes;
    else if (k == "ring_ctas") *value = c->ring_ctas;
    else if (k == "timeout_ns") *value = c->timeout_ns;
    else if (k == "fault_skip_rank") *value = c->fault_skip_rank;
    else if (k == "copy_variant") *value = c->copy_variant;
    else if (k == "copy_order") *value = c->copy_order;
    else if (k == "direct_pack") *value = c->direct_pack;
    else if (k == "l2_hint") *value = c->l2_hint;
    else if (k == "direct_ctas_per_sm") *value = c->direct_ctas_per_sm;
    else if (k == "moe_tma") *value = c->moe_tma;
    else if (k == "moe_fused") *value = c->moe_fused;
    else if (k == "ring_task_bytes") *value = c->ring_task_bytes;
    else if (k == "trace") *value = c->trace;
    else return fail(COLL_ERR_INVALID_ARG, "unknown option " + k);
    return COLL_OK;
}

coll_status_t sim_comm_get_async_error(sim_comm_t c, coll_status_t* out) {
    if (!c || !out) return fail(COLL_ERR_INVALID_ARG, "null argument");
    *out = coll_status_t(static_cast<volatile uint32_t*>(c->host_words)[0]);
    return COLL_OK;
}

coll_status_t sim_comm_abort(sim_comm_t c) {
    if (!c) return fail(COLL_ERR_INVALID_ARG, "null communicator");
    static_cast<volatile uint32_t*>(c->host_words)[1] = 1u;
    return COLL_OK;
}

coll_status_t sim_comm_reset(sim_comm_t c) {
    if (!c) return fail(COLL_ERR_INVALID_ARG, "null communicator");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "sim_comm_reset: device synchronisation");
    e = cudaMemset(c->dstate, 0, sizeof(DevState));
    if (e == cudaSuccess && c->flags) e = cudaMemset(c->flags, 0, c->flags_cap * sizeof(unsigned long long));
    if (e == cudaSuccess && c->moe_acc) e = cudaMemset(c->moe_acc, 0, c->moe_acc_cap * sizeof(int32_t));
    for (const auto& ra : c->retired_acc)
        if (e == cudaSuccess) e = cudaMemset(ra.first, 0, ra.second * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "sim_comm_reset");
    c->epoch = 0;
    volatile uint32_t* hw = c->host_words;
    hw[0] = 0u;
    hw[1] = 0u;
    return COLL_OK;
}

coll_status_t sim_comm_launch_count(sim_comm_t c, unsigned long long* out) {
    if (!c || !out) return fail(COLL_ERR_INVALID_ARG, "null argument");
    *out = c->launches;
    return COLL_OK;
}

// ---- collectives -------------------------------------------------------------------------------

static coll_status_t coll_allreduce_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op,
                                         coll_algo_t algo, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if ((st = check_reduce_args(dt, op)) != COLL_OK || (st = check_algo(algo, true)) != COLL_OK) return st;
    if ((algo == COLL_ALGO_RD || algo == COLL_ALGO_HD || algo == COLL_ALGO_RD_LL) && (c->p & (c->p - 1)))
        return fail(COLL_ERR_UNSUPPORTED, "recursive doubling / halving-doubling need p a power of two");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_ALLREDUCE, b, n, dt, op, 0, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const int p = c->p;
    const size_t d = dtype_bytes(dt), bytes = n * d;
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], bytes, d, "send")) != COLL_OK) return st;
        if ((st = check_ptr(b.recv[r], bytes, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + bytes, false, r});
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + bytes, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_SAME, 0)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (algo == COLL_ALGO_DIRECT || p == 1) return run_direct_reduce(c, b, n, dt, op, MODE_ALLREDUCE, 0, s);
    if (algo == COLL_ALGO_RD) return run_butterfly(c, b, n, dt, op, BFLY_RD, s);
    if (algo == COLL_ALGO_HD) return run_butterfly(c, b, n, dt, op, BFLY_HD, s);
    if (algo == COLL_ALGO_TREE || algo == COLL_ALGO_DBTREE) return run_tree(c, b, n, dt, op, algo == COLL_ALGO_DBTREE, s);
    if (algo == COLL_ALGO_RING_LL) return run_ring_ll(c, b, n, dt, op, s);
    if (algo == COLL_ALGO_RD_LL) return run_rd_ll(c, b, n, dt, op, s);
    if (algo == COLL_ALGO_TREE_LL || algo == COLL_ALGO_DBTREE_LL)
        return run_tree_ll(c, b, n, dt, op, algo == COLL_ALGO_DBTREE_LL, s);
    RingPlan pl;
    pl.kind = RING_ALLREDUCE;
    pl.seg = (n + size_t(p) - 1) / size_t(p);
    pl.chunk = size_t(c->chunk_bytes) / 4;  // chunk counted in the fp32/int32 partial type
    pl.nch = chunks_of(pl.seg, pl.chunk);
    pl.nsteps = uint32_t(2 * (p - 1));
    pl.rps = uint32_t(p);
    pl.needs_stage = true;
    return run_ring(c, b, pl, n, dt, op, 0, s);
}

static coll_status_t coll_reduce_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op, int root,
                                      coll_algo_t algo, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if ((st = check_reduce_args(dt, op)) != COLL_OK || (st = check_algo(algo)) != COLL_OK) return st;
    const int p = c->p;
    if (root < 0 || root >= p) return fail(COLL_ERR_INVALID_ARG, "root must be a rank index in [0, p)");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_REDUCE, b, n, dt, op, root, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), bytes = n * d;
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], bytes, d, "send")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + bytes, false, r});
    }
    if ((st = check_ptr(b.recv[root], bytes, d, "root recv")) != COLL_OK) return st;
    rs.push_back({uintptr_t(b.recv[root]), uintptr_t(b.recv[root]) + bytes, true, root});
    if ((st = check_ranges(rs, INPLACE_SAME, 0)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Only recv[root] is touched; the kernels are handed a copy of the array with the others null.
    std::vector<void*> recv(p, nullptr);
    recv[root] = b.recv[root];
    coll_bufs_t bb{b.send, recv.data()};
    if (algo == COLL_ALGO_DIRECT || p == 1) return run_direct_reduce(c, bb, n, dt, op, MODE_REDUCE, root, s);
    RingPlan pl;
    pl.kind = RING_REDUCE;
    pl.seg = n;
    pl.chunk = size_t(c->chunk_bytes) / 4;
    pl.nch = chunks_of(n, pl.chunk);
    pl.nsteps = uint32_t(p - 1);
    pl.rps = 1;
    pl.needs_stage = true;
    return run_ring(c, bb, pl, n, dt, op, root, s);
}

static coll_status_t coll_broadcast_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, int root,
                                         coll_algo_t algo, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if ((st = check_algo(algo)) != COLL_OK) return st;
    const int p = c->p;
    if (root < 0 || root >= p) return fail(COLL_ERR_INVALID_ARG, "root must be a rank index in [0, p)");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_BCAST, b, n, dt, COLL_SUM, root, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), bytes = n * d;
    std::vector<Range> rs;
    if ((st = check_ptr(b.send[root], bytes, d, "root send")) != COLL_OK) return st;
    rs.push_back({uintptr_t(b.send[root]), uintptr_t(b.send[root]) + bytes, false, root});
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.recv[r], bytes, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + bytes, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_SAME, 0)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<const void*> send(p, nullptr);
    send[root] = b.send[root];
    coll_bufs_t bb{send.data(), b.recv};
    if (algo == COLL_ALGO_DIRECT || p == 1) return run_copy(c, bb, COPY_BCAST, n, dt, root, false, s);
    RingPlan pl;
    pl.kind = RING_BCAST;
    pl.seg = n;
    pl.chunk = size_t(c->chunk_bytes) / d;
    pl.nch = chunks_of(n, pl.chunk);
    pl.nsteps = uint32_t(p);
    pl.rps = 1;
    pl.needs_stage = false;
    return run_ring(c, bb, pl, n, dt, COLL_SUM, root, s);
}

static coll_status_t coll_reduce_scatter_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op,
                                              coll_algo_t algo, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if ((st = check_reduce_args(dt, op)) != COLL_OK || (st = check_algo(algo, false, true)) != COLL_OK) return st;
    const int p = c->p;
    if (n % size_t(p) != 0) return fail(COLL_ERR_INVALID_ARG, "ReduceScatter needs n divisible by p");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_REDUCE_SCATTER, b, n, dt, op, 0, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), m = n / size_t(p);
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], n * d, d, "send")) != COLL_OK) return st;
        if ((st = check_ptr(b.recv[r], m * d, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + n * d, false, r});
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + m * d, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_RS, m * d)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (algo == COLL_ALGO_DIRECT || p == 1) return run_direct_reduce(c, b, n, dt, op, MODE_REDUCE_SCATTER, 0, s);
    if (algo == COLL_ALGO_RING_LL) return run_ring_ll(c, b, n, dt, op, s, LL_RING_RS);
    RingPlan pl;
    pl.kind = RING_REDUCE_SCATTER;
    pl.seg = m;
    pl.chunk = size_t(c->chunk_bytes) / 4;
    pl.nch = chunks_of(m, pl.chunk);
    pl.nsteps = uint32_t(p - 1);
    pl.rps = uint32_t(p);
    pl.needs_stage = true;
    return run_ring(c, b, pl, n, dt, op, 0, s);
}

static coll_status_t coll_allgather_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_algo_t algo,
                                         coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if ((st = check_algo(algo, false, true)) != COLL_OK) return st;
    const int p = c->p;
    if (n % size_t(p) != 0) return fail(COLL_ERR_INVALID_ARG, "AllGather needs n divisible by p");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_ALLGATHER, b, n, dt, COLL_SUM, 0, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), m = n / size_t(p);
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], m * d, d, "send")) != COLL_OK) return st;
        if ((st = check_ptr(b.recv[r], n * d, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + m * d, false, r});
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + n * d, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_AG, m * d)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (algo == COLL_ALGO_DIRECT || p == 1) return run_copy(c, b, COPY_ALLGATHER, m, dt, 0, true, s);
    if (algo == COLL_ALGO_RING_LL) return run_ring_ll(c, b, n, dt, COLL_SUM, s, LL_RING_AG);
    RingPlan pl;
    pl.kind = RING_ALLGATHER;
    pl.seg = m;
    pl.chunk = size_t(c->chunk_bytes) / d;
    pl.nch = chunks_of(m, pl.chunk);
    pl.nsteps = uint32_t(p);
    pl.rps = uint32_t(p);
    pl.needs_stage = false;
    return run_ring(c, b, pl, n, dt, COLL_SUM, 0, s);
}

static coll_status_t coll_alltoall_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_algo_t algo,
                                        coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if ((st = check_algo(algo)) != COLL_OK) return st;
    const int p = c->p;
    if (n % size_t(p) != 0) return fail(COLL_ERR_INVALID_ARG, "All-to-All needs n divisible by p");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_ALLTOALL, b, n, dt, COLL_SUM, 0, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), m = n / size_t(p);
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], n * d, d, "send")) != COLL_OK) return st;
        if ((st = check_ptr(b.recv[r], n * d, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + n * d, false, r});
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + n * d, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_NONE, 0)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (algo == COLL_ALGO_DIRECT || p == 1) return run_copy(c, b, COPY_ALLTOALL, m, dt, 0, true, s);
    RingPlan pl;
    pl.kind = RING_ALLTOALL;
    pl.seg = m;
    pl.chunk = size_t(c->chunk_bytes) / d;
    pl.nch = chunks_of(m, pl.chunk);
    pl.nsteps = uint32_t(p);
    pl.rps = uint32_t(p);
    pl.needs_stage = false;
    return run_ring(c, b, pl, n, dt, COLL_SUM, 0, s);
}

static coll_status_t coll_scatter_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, int root,
                                       coll_algo_t algo, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if ((st = check_algo(algo)) != COLL_OK) return st;
    if (algo != COLL_ALGO_DIRECT) return fail(COLL_ERR_UNSUPPORTED, "Scatter has the direct path only");
    const int p = c->p;
    if (root < 0 || root >= p) return fail(COLL_ERR_INVALID_ARG, "root must be a rank index in [0, p)");
    if (n % size_t(p) != 0) return fail(COLL_ERR_INVALID_ARG, "Scatter needs n divisible by p");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_SCATTER, b, n, dt, COLL_SUM, root, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), m = n / size_t(p);
    std::vector<Range> rs;
    if ((st = check_ptr(b.send[root], n * d, d, "root send")) != COLL_OK) return st;
    rs.push_back({uintptr_t(b.send[root]), uintptr_t(b.send[root]) + n * d, false, root});
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.recv[r], m * d, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + m * d, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_RS, m * d)) != COLL_OK) return st;  // recv[root] = send[root] + root·m
    std::vector<const void*> send(p, nullptr);
    send[root] = b.send[root];
    coll_bufs_t bb{send.data(), b.recv};
    return run_copy(c, bb, COPY_SCATTER, m, dt, root, false, static_cast<cudaStream_t>(stream));
}

static coll_status_t coll_gather_impl(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, int root,
                                      coll_algo_t algo, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if ((st = check_algo(algo)) != COLL_OK) return st;
    if (algo != COLL_ALGO_DIRECT) return fail(COLL_ERR_UNSUPPORTED, "Gather has the direct path only");
    const int p = c->p;
    if (root < 0 || root >= p) return fail(COLL_ERR_INVALID_ARG, "root must be a rank index in [0, p)");
    if (n % size_t(p) != 0) return fail(COLL_ERR_INVALID_ARG, "Gather needs n divisible by p");
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (c->rank >= 0) {
        if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
        return rank_collective(c, RK_GATHER, b, n, dt, COLL_SUM, root, algo, static_cast<cudaStream_t>(stream));
    }
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), m = n / size_t(p);
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], m * d, d, "send")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + m * d, false, r});
    }
    if ((st = check_ptr(b.recv[root], n * d, d, "root recv")) != COLL_OK) return st;
    rs.push_back({uintptr_t(b.recv[root]), uintptr_t(b.recv[root]) + n * d, true, root});
    if ((st = check_ranges(rs, INPLACE_AG, m * d)) != COLL_OK) return st;  // send[root] = recv[root] + root·m
    std::vector<void*> recv(p, nullptr);
    recv[root] = b.recv[root];
    coll_bufs_t bb{b.send, recv.data()};
    return run_copy(c, bb, COPY_GATHER, m, dt, root, true, static_cast<cudaStream_t>(stream));
}

static coll_status_t coll_alltoallv_impl(sim_comm_t c, coll_bufs_t b, const long long* counts_dev,
                                         const long long* send_cap, const long long* recv_cap, coll_dtype_t dt,
                                         coll_algo_t algo, coll_stream_t stream, long long* recv_counts_dev) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if ((st = check_algo(algo)) != COLL_OK) return st;
    if (!counts_dev || !send_cap || !recv_cap) return fail(COLL_ERR_INVALID_ARG, "null counts or capacities");
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    if (reinterpret_cast<uintptr_t>(counts_dev) % 8 != 0 ||
        (recv_counts_dev && reinterpret_cast<uintptr_t>(recv_counts_dev) % 8 != 0))
        return fail(COLL_ERR_INVALID_ARG, "count arrays must be 8-byte aligned");
    const int p = c->p;
    const size_t d = dtype_bytes(dt);
    std::vector<Range> rs;
    const bool view = c->rank >= 0;  // a rank view writes only its own output
    for (int r = 0; r < p; ++r) {
        if (send_cap[r] < 0 || recv_cap[r] < 0) return fail(COLL_ERR_INVALID_ARG, "negative capacity");
        if ((st = check_count(size_t(send_cap[r]), "send_cap")) != COLL_OK ||
            (st = check_count(size_t(recv_cap[r]), "recv_cap")) != COLL_OK)
            return st;
        const size_t sb = size_t(send_cap[r]) * d, rb = size_t(recv_cap[r]) * d;
        if ((st = check_ptr(b.send[r], sb, d, "send")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + sb, false, r});
        if (view && r != c->rank) continue;
        if ((st = check_ptr(b.recv[r], rb, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + rb, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_NONE, 0)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (view) {
        if (algo != COLL_ALGO_DIRECT)
            return fail(COLL_ERR_UNSUPPORTED, "a rank view runs the direct path only");
        // the blocks bound for this rank, pulled from every source (each rank holds the whole count
        // matrix, so every rank computes the same displacements and capacity decision)
        std::vector<void*> recv(p, nullptr);
        recv[c->rank] = b.recv[c->rank];
        return run_copy(c, coll_bufs_t{b.send, recv.data()}, COPY_ALLTOALLV, 0, dt, 0, true, s, counts_dev, send_cap,
                        recv_cap, recv_counts_dev, 0, c->rank);
    }
    if (algo == COLL_ALGO_DIRECT || p == 1)
        return run_copy(c, b, COPY_ALLTOALLV, 0, dt, 0, true, s, counts_dev, send_cap, recv_cap, recv_counts_dev);
    RingPlan pl;
    pl.kind = RING_ALLTOALLV;
    pl.seg = 0;
    pl.chunk = size_t(c->chunk_bytes) / d;
    pl.nch = 0;  // from the largest count, on the device
    pl.nsteps = uint32_t(p);
    pl.rps = uint32_t(p);
    pl.needs_stage = false;
    return run_ring(c, b, pl, 0, dt, COLL_SUM, 0, s, counts_dev, send_cap, recv_cap, recv_counts_dev);
}

}  // extern "C"

// ---- MoE dispatch and combine -------------------------------------------------------------------

namespace {

// Shape checks shared by dispatch and combine.
coll_status_t check_moe_shape(sim_comm* c, size_t tokens, int k, size_t hidden, int experts) {
    const int p = c->p;
    if (k < 1 || k > kMoeMaxTopk) return fail(COLL_ERR_INVALID_ARG, "k must be in [1, 32]");
    if (experts < p || experts % p != 0 || experts > kMoeMaxExperts)
        return fail(COLL_ERR_INVALID_ARG, "experts must be a multiple of p in [p, 4096]");
    if (hidden == 0) return fail(COLL_ERR_INVALID_ARG, "hidden must be positive");
    if (check_count(hidden, "hidden") != COLL_OK) return COLL_ERR_INVALID_ARG;
    if (tokens > size_t(INT32_MAX) / size_t(k)) return fail(COLL_ERR_INVALID_ARG, "tokens * k must fit in int32");
    return check_rows(tokens, hidden, "tokens");
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" {

static coll_status_t coll_moe_dispatch_impl(sim_comm_t c, const void* const* x, const int32_t* const* topk_idx,
                                            size_t tokens, int k, size_t hidden, int experts, coll_dtype_t dt,
                                            void* const* recv, size_t recv_cap_rows, int32_t* const* route_pos,
                                            long long* expert_counts_dev, long long* recv_counts_dev,
                                            coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if (c->rank >= 0 && !c->moe_fused)
        return fail(COLL_ERR_UNSUPPORTED, "a rank view's MoE dispatch runs the fused kernel only (option moe_fused 1)");
    if ((st = check_moe_shape(c, tokens, k, hidden, experts)) != COLL_OK) return st;
    if (recv_cap_rows > size_t(INT32_MAX)) return fail(COLL_ERR_INVALID_ARG, "recv_cap_rows must fit in int32");
    if ((st = check_rows(recv_cap_rows, hidden, "recv_cap_rows")) != COLL_OK) return st;
    if (!x || !topk_idx || !recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    if ((expert_counts_dev && reinterpret_cast<uintptr_t>(expert_counts_dev) % 8 != 0) ||
        (recv_counts_dev && reinterpret_cast<uintptr_t>(recv_counts_dev) % 8 != 0))
        return fail(COLL_ERR_INVALID_ARG, "count arrays must be 8-byte aligned");
    const int p = c->p;
    const size_t d = dtype_bytes(dt), row = hidden * d, A = tokens * size_t(k);
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(x[r], tokens * row, d, "token")) != COLL_OK) return st;
        if ((st = check_ptr(topk_idx[r], A * 4, 4, "expert id")) != COLL_OK) return st;
        rs.push_back({uintptr_t(x[r]), uintptr_t(x[r]) + tokens * row, false, r});
        rs.push_back({uintptr_t(topk_idx[r]), uintptr_t(topk_idx[r]) + A * 4, false, r});
        if (c->rank >= 0 && r != c->rank) continue;  // a rank view writes only its own outputs
        if ((st = check_ptr(recv[r], recv_cap_rows * row, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(recv[r]), uintptr_t(recv[r]) + recv_cap_rows * row, true, r});
        if (route_pos) {
            if ((st = check_ptr(route_pos[r], A * 4, 4, "route_pos")) != COLL_OK) return st;
            rs.push_back({uintptr_t(route_pos[r]), uintptr_t(route_pos[r]) + A * 4, true, r});
        }
    }
    if ((st = check_ranges(rs, INPLACE_NONE, 0)) != COLL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) {  // nothing routed: only the count outputs change
        cudaError_t e = cudaSuccess;
        if (expert_counts_dev) e = cudaMemsetAsync(expert_counts_dev, 0, size_t(p) * experts * sizeof(long long), s);
        if (e == cudaSuccess && recv_counts_dev) e = cudaMemsetAsync(recv_counts_dev, 0, size_t(p) * sizeof(long long), s);
        return e == cudaSuccess ? COLL_OK : cuda_fail(e, "cudaMemsetAsync(MoE counts)");
    }
    MoeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.k = k;
    a.E = experts;
    a.E_loc = experts / p;
    a.elem_bytes = int(d);
    a.T = tokens;
    a.H = hidden;
    a.A = A;
    a.cap_rows = recv_cap_rows;
    a.ntiles = uint32_t((A + kMoeTile - 1) / kMoeTile);
    a.view_rank = c->rank;
    for (int r = 0; r < p; ++r) {
        const bool own = c->rank < 0 || r == c->rank;
        a.src[r] = x[r];
        a.idx[r] = topk_idx[r];
        a.dst[r] = own ? recv[r] : nullptr;
        a.pos[r] = own && route_pos ? route_pos[r] : nullptr;
    }
    // scratch: tile counts [p][ntiles][E], in-tile ranks [p][A], totals and first rows [p][E] each,
    // the count matrix [p][p]
    const size_t b_hist = align_up(size_t(p) * a.ntiles * experts * 4, 256);
    const size_t b_rank = align_up(size_t(p) * A * 4, 256);
    const size_t b_pe = align_up(size_t(p) * experts * 4, 256);
    const size_t b_pp = align_up(size_t(p) * p * 4, 256);
    if ((st = ensure_moe(c, b_hist + b_rank + 2 * b_pe + b_pp)) != COLL_OK) return st;
    a.tile_hist = reinterpret_cast<int32_t*>(c->moe);
    a.rank_in_tile = reinterpret_cast<int32_t*>(c->moe + b_hist);
    a.cnt = reinterpret_cast<int32_t*>(c->moe + b_hist + b_rank);
    a.base = reinterpret_cast<int32_t*>(c->moe + b_hist + b_rank + b_pe);
    a.cmat = reinterpret_cast<int32_t*>(c->moe + b_hist + b_rank + 2 * b_pe);
    if (c->moe_fused) {
        if ((st = ensure_moe_acc(c, size_t(p) * experts)) != COLL_OK) return st;
        a.acc = c->moe_acc;
    }
    a.expert_counts_out = expert_counts_dev;
    a.recv_counts_out = recv_counts_dev;
    a.tma = int(c->moe_tma);
    a.fused = int(c->moe_fused);
    a.skip_cta = int(c->fault_skip_rank);
    a.timeout_ns = uint64_t(c->timeout_ns);
    a.st = c->dstate;
    a.ctl = make_ctl(c);
    int launched = 0;
    cudaError_t e = launch_moe_dispatch(a, c->num_sms, s, &launched);
    if (e != cudaSuccess) return cuda_fail(e, "MoE dispatch launch");
    c->launches += unsigned(launched);
    return COLL_OK;
}

static coll_status_t coll_moe_combine_impl(sim_comm_t c, const void* const* y, size_t y_rows,
                                           const int32_t* const* topk_idx, const int32_t* const* route_pos,
                                           const float* const* topk_weight, const void* const* residual,
                                           size_t tokens, int k, size_t hidden, int experts, coll_dtype_t dt,
                                           void* const* out, coll_stream_t stream) {
    coll_status_t st = check_usable(c);
    if (st != COLL_OK) return st;
    if (!valid_dtype(dt)) return fail(COLL_ERR_INVALID_ARG, "unknown dtype");
    if (dt == COLL_INT32) return fail(COLL_ERR_UNSUPPORTED, "the weighted combine needs fp32 or bf16 rows");
    if ((st = check_moe_shape(c, tokens, k, hidden, experts)) != COLL_OK) return st;
    if ((st = check_rows(y_rows, hidden, "y_rows")) != COLL_OK) return st;
    if (!y || !topk_idx || !route_pos || !topk_weight || !out) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    if (tokens == 0) return COLL_OK;
    const int p = c->p;
    const size_t d = dtype_bytes(dt), row = hidden * d, A = tokens * size_t(k);
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(y[r], y_rows * row, d, "expert output")) != COLL_OK) return st;
        rs.push_back({uintptr_t(y[r]), uintptr_t(y[r]) + y_rows * row, false, r});
        if (c->rank >= 0 && r != c->rank) continue;  // a rank view combines only its own tokens
        if ((st = check_ptr(topk_idx[r], A * 4, 4, "expert id")) != COLL_OK) return st;
        if ((st = check_ptr(route_pos[r], A * 4, 4, "route_pos")) != COLL_OK) return st;
        if ((st = check_ptr(topk_weight[r], A * 4, 4, "gate weight")) != COLL_OK) return st;
        if ((st = check_ptr(out[r], tokens * row, d, "out")) != COLL_OK) return st;
        rs.push_back({uintptr_t(topk_idx[r]), uintptr_t(topk_idx[r]) + A * 4, false, r});
        rs.push_back({uintptr_t(route_pos[r]), uintptr_t(route_pos[r]) + A * 4, false, r});
        rs.push_back({uintptr_t(topk_weight[r]), uintptr_t(topk_weight[r]) + A * 4, false, r});
        rs.push_back({uintptr_t(out[r]), uintptr_t(out[r]) + tokens * row, true, r});
        if (residual && (st = check_ptr(residual[r], tokens * row, d, "residual")) != COLL_OK) return st;
    }
    if ((st = check_ranges(rs, INPLACE_NONE, 0)) != COLL_OK) return st;
    // a residual may be its own rank's output (out = residual + Σ w y, element by element), and
    // must not overlap any other output
    for (int r = 0; residual && r < p; ++r) {
        if (c->rank >= 0 && r != c->rank) continue;
        const Range res{uintptr_t(residual[r]), uintptr_t(residual[r]) + tokens * row, false, r};
        for (int q = 0; q < p; ++q) {
            if (c->rank >= 0 && q != c->rank) continue;
            const Range o{uintptr_t(out[q]), uintptr_t(out[q]) + tokens * row, true, q};
            if (overlap(res, o) && !(q == r && res.lo == o.lo))
                return fail(COLL_ERR_INVALID_ARG, "a residual overlaps an output other than its own rank's");
        }
    }
    MoeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.k = k;
    a.E = experts;
    a.E_loc = experts / p;
    a.elem_bytes = int(d);
    a.has_res = residual ? 1 : 0;
    a.T = tokens;
    a.H = hidden;
    a.A = A;
    a.cap_rows = y_rows;
    a.view_rank = c->rank;
    for (int r = 0; r < p; ++r) {
        a.src[r] = y[r];
        if (c->rank >= 0 && r != c->rank) continue;
        a.idx[r] = topk_idx[r];
        a.pos[r] = const_cast<int32_t*>(route_pos[r]);
        a.w[r] = topk_weight[r];
        a.dst[r] = out[r];
        a.res[r] = residual ? residual[r] : nullptr;
    }
    a.st = c->dstate;
    a.ctl = make_ctl(c);
    cudaError_t e = launch_moe_combine(a, int(dt), c->num_sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "MoE combine launch");
    c->launches += 1;
    return COLL_OK;
}

}  // extern "C"

// =================================================================================================
// Ring AllReduce without any allocation.
//
// Some callers cannot call cudaMalloc: code inside a memory-pool or allocator implementation (it
// must not re-enter the allocator it implements), a process that must not grow its device footprint
// after start-up, or code where a framework forbids allocation. For them this entry point runs the
// same ring AllReduce kernel, with the same schedule and tiling, as coll_allreduce(...,
// COLL_ALGO_RING, ...) with default options, on a fixed scratch area that is part of the library
// image: a file-scope device array of kStaticScratchBytes. No communicator is created and nothing is
// allocated or freed per call.
//
// The array lives in device memory of every GPU that loads this library until the process exits.
// In host code its name is only a host-side handle, never a device address: a kernel given it
// would fault, or silently use the wrong memory where the GPU can reach host memory. Its device
// address is therefore looked up once per device, with that device current, by the first call on
// that device (cudaGetSymbolAddress); that first call should come before any stream capture.
// Every call shares the array and it keeps the last call's contents: each call clears the control
// words and chunk flags it needs on its stream before the kernel, and calls whose work overlaps on
// the GPU (other streams, other host threads) race on the array and must be ordered by the caller.
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxStaticDevices = 64;

// An integer option from the environment, or `dflt` when the variable is unset, not a whole
// number, or outside [lo, hi].
long long env_option(const char* name, long long dflt, long long lo, long long hi) {
    const char* v = std::getenv(name);
    if (!v || !*v) return dflt;
    char* end = nullptr;
    const long long x = std::strtoll(v, &end, 0);
    return (end && *end == 0 && x >= lo && x <= hi) ? x : dflt;
}
std::mutex g_static_mu;
char* g_static_base[kMaxStaticDevices] = {};
int g_static_sms[kMaxStaticDevices] = {};
int g_static_ctas[kMaxStaticDevices] = {};

}  // namespace

extern "C" coll_status_t coll_allreduce_ring_noalloc(int p, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op,
                                                     int* async_status_dev, coll_stream_t stream) {
    coll_status_t st;
    if (p < 2 || p > SIM_COMM_MAX_RANKS) return fail(COLL_ERR_INVALID_ARG, "p must be in [2, 64]");
    if ((st = check_reduce_args(dt, op)) != COLL_OK) return st;
    if (n == 0) return COLL_OK;
    if ((st = check_count(n, "n")) != COLL_OK) return st;
    if (!b.send || !b.recv) return fail(COLL_ERR_INVALID_ARG, "null buffer array");
    const size_t d = dtype_bytes(dt), bytes = n * d;
    std::vector<Range> rs;
    for (int r = 0; r < p; ++r) {
        if ((st = check_ptr(b.send[r], bytes, d, "send")) != COLL_OK) return st;
        if ((st = check_ptr(b.recv[r], bytes, d, "recv")) != COLL_OK) return st;
        rs.push_back({uintptr_t(b.send[r]), uintptr_t(b.send[r]) + bytes, false, r});
        rs.push_back({uintptr_t(b.recv[r]), uintptr_t(b.recv[r]) + bytes, true, r});
    }
    if ((st = check_ranges(rs, INPLACE_SAME, 0)) != COLL_OK) return st;

    // Layout of the scratch: control words, chunk flags, then one partial buffer per rank.
    const size_t seg = (n + size_t(p) - 1) / size_t(p);
    const size_t chunk = (size_t(1) << 20) / 4;
    const uint32_t nch = chunks_of(seg, chunk);
    const uint32_t nsteps = uint32_t(2 * (p - 1));
    const size_t ctl_bytes = round_up(sizeof(DevState) + 8, 256);
    const size_t flag_bytes = round_up(size_t(nsteps) * p * nch * sizeof(unsigned long long), 256);
    const size_t stride = round_up(n * 4, 256);
    const size_t need = ctl_bytes + flag_bytes + size_t(p) * stride;
    if (need > kStaticScratchBytes)
        return fail(COLL_ERR_INVALID_ARG, "coll_allreduce_ring_noalloc needs " + std::to_string(need) +
                                              " bytes of scratch; its static scratch holds " +
                                              std::to_string(kStaticScratchBytes) + " (p * n * 4 must stay below ~32 MiB)");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxStaticDevices) return fail(COLL_ERR_UNSUPPORTED, "device ordinal above 63");
    char* base;
    int ctas;
    {
        std::lock_guard<std::mutex> lock(g_static_mu);
        if (!g_static_base[dev]) {
            void* ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_static_scratch);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
            e = cudaDeviceGetAttribute(&g_static_sms[dev], cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
            g_static_ctas[dev] = ring_max_ctas(g_static_sms[dev]);
            g_static_base[dev] = static_cast<char*>(ptr);
        }
        base = g_static_base[dev];
        ctas = g_static_ctas[dev];
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the control words and flags must start at zero for this call
    e = cudaMemsetAsync(base, 0, ctl_bytes + flag_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(static scratch)");

    RingArgs a;
    std::memset(&a, 0, sizeof(a));
    fill_ptrs(a.ptrs, b, p, true, true);
    a.p = p;
    a.kind = RING_ALLREDUCE;
    a.root = 0;
    a.n = n;
    a.seg = seg;
    a.chunk = chunk;
    // the same tiling as coll_allreduce(..., COLL_ALGO_RING) with default options
    ring_tiles(std::min(chunk, seg), 4, default_task_bytes(n * 4), &a.tile, &a.ntile);
    a.elem_bytes = int(d);
    a.nch = nch;
    a.nsteps = nsteps;
    a.ranks_per_step = uint32_t(p);
    a.epoch = 1;
    a.scale = (op == COLL_AVG) ? 1.0f / float(p) : 1.0f;
    a.skip_rank = int(env_option("SIMCOMM_FAULT_SKIP_RANK", -1, -1, p - 1));
    a.timeout_ns = uint64_t(env_option("SIMCOMM_TIMEOUT_NS", 2000000000LL, 1000, LLONG_MAX));
    a.st = reinterpret_cast<DevState*>(base);
    a.ctl.status = &a.st->status;

    a.ctl.host_status = reinterpret_cast<uint32_t*>(base + sizeof(DevState));
    a.ctl.abort_flag = reinterpret_cast<uint32_t*>(base + sizeof(DevState) + 4);
    a.ctl.abort_clock = &a.st->abort_clock;
    a.flags = reinterpret_cast<unsigned long long*>(base + ctl_bytes);
    a.stage = base + ctl_bytes + flag_bytes;
    a.stage_stride = stride;
    bool vec = (seg * d) % 16 == 0 && (seg * 4) % 16 == 0 && (chunk * d) % 16 == 0;
    for (int r = 0; r < p; ++r) vec = vec && aligned16(a.ptrs.send[r]) && aligned16(a.ptrs.recv[r]);
    a.vec = vec ? 1 : 0;
    const size_t tasks = size_t(nsteps) * p * nch * a.ntile;
    if (tasks < size_t(ctas)) ctas = int(std::max<size_t>(tasks, 1));
    e = launch_ring(a, dt, op, ctas, s);
    if (e != cudaSuccess) return cuda_fail(e, "ring executor launch");
    if (async_status_dev) {
        e = cudaMemcpyAsync(async_status_dev, &a.st->status, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(status)");
    }
    return COLL_OK;
}

// ---- HBM access-pattern probe ----------------------------------------------------------------------

extern "C" coll_status_t sim_hbm_probe(int kind, void* dst, const void* src, size_t bytes, int ctas_per_sm,
                                       coll_stream_t stream) {
    if (kind < PROBE_LOAD || kind > PROBE_BULK_FANOUT) return fail(COLL_ERR_INVALID_ARG, "unknown probe kind");
    if (ctas_per_sm < 0 || ctas_per_sm > 32) return fail(COLL_ERR_INVALID_ARG, "ctas_per_sm must be in [0, 32]");
    if (bytes == 0) return COLL_OK;
    if (check_probe_bytes(bytes) != COLL_OK) return COLL_ERR_INVALID_ARG;
    if (kind == PROBE_BULK_FANOUT && (bytes % (32 * 1024) != 0 || bytes > (size_t(1) << 40)))
        return fail(COLL_ERR_INVALID_ARG, "fan-out probe bytes must be a multiple of 32 KiB, at most 2^40");
    const bool reads = kind == PROBE_LOAD || kind == PROBE_COPY || kind == PROBE_BULK_FANOUT;
    const bool writes = kind != PROBE_LOAD;
    const size_t dst_bytes = kind == PROBE_BULK_FANOUT ? bytes * kProbeFanCopies : bytes;
    if ((reads && (!src || uintptr_t(src) % 256 != 0)) || (writes && (!dst || uintptr_t(dst) % 256 != 0)))
        return fail(COLL_ERR_INVALID_ARG, "probe buffers must be non-null and 256-byte aligned");
    if (reads && writes && overlap(Range{uintptr_t(src), uintptr_t(src) + bytes, false, 0},
                                   Range{uintptr_t(dst), uintptr_t(dst) + dst_bytes, true, 0}))
        return fail(COLL_ERR_INVALID_ARG, "probe buffers overlap");
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "probe: device query");
    e = launch_probe(kind, dst, src, bytes, ctas_per_sm, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? COLL_OK : cuda_fail(e, "probe launch");
}

// ---- traced entry points --------------------------------------------------------------------------

extern "C" {

coll_status_t coll_allreduce(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op, coll_algo_t algo,
                             coll_stream_t stream) {
    TraceScope ts(c, "allreduce", n, int(dt), int(op), -1, int(algo), stream);
    return ts.done(coll_allreduce_impl(c, b, n, dt, op, algo, stream));
}

coll_status_t coll_reduce(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op, int root,
                          coll_algo_t algo, coll_stream_t stream) {
    TraceScope ts(c, "reduce", n, int(dt), int(op), root, int(algo), stream);
    return ts.done(coll_reduce_impl(c, b, n, dt, op, root, algo, stream));
}

coll_status_t coll_broadcast(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, int root, coll_algo_t algo,
                             coll_stream_t stream) {
    TraceScope ts(c, "broadcast", n, int(dt), -1, root, int(algo), stream);
    return ts.done(coll_broadcast_impl(c, b, n, dt, root, algo, stream));
}

coll_status_t coll_reduce_scatter(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_op_t op,
                                  coll_algo_t algo, coll_stream_t stream) {
    TraceScope ts(c, "reduce_scatter", n, int(dt), int(op), -1, int(algo), stream);
    return ts.done(coll_reduce_scatter_impl(c, b, n, dt, op, algo, stream));
}

coll_status_t coll_allgather(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_algo_t algo,
                             coll_stream_t stream) {
    TraceScope ts(c, "allgather", n, int(dt), -1, -1, int(algo), stream);
    return ts.done(coll_allgather_impl(c, b, n, dt, algo, stream));
}

coll_status_t coll_alltoall(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, coll_algo_t algo,
                            coll_stream_t stream) {
    TraceScope ts(c, "alltoall", n, int(dt), -1, -1, int(algo), stream);
    return ts.done(coll_alltoall_impl(c, b, n, dt, algo, stream));
}

coll_status_t coll_scatter(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, int root, coll_algo_t algo,
                           coll_stream_t stream) {
    TraceScope ts(c, "scatter", n, int(dt), -1, root, int(algo), stream);
    return ts.done(coll_scatter_impl(c, b, n, dt, root, algo, stream));
}

coll_status_t coll_gather(sim_comm_t c, coll_bufs_t b, size_t n, coll_dtype_t dt, int root, coll_algo_t algo,
                          coll_stream_t stream) {
    TraceScope ts(c, "gather", n, int(dt), -1, root, int(algo), stream);
    return ts.done(coll_gather_impl(c, b, n, dt, root, algo, stream));
}

coll_status_t coll_alltoallv(sim_comm_t c, coll_bufs_t b, const long long* counts_dev, const long long* send_cap,
                             const long long* recv_cap, coll_dtype_t dt, coll_algo_t algo, coll_stream_t stream,
                             long long* recv_counts_dev) {
    TraceScope ts(c, "alltoallv", 0, int(dt), -1, -1, int(algo), stream);
    return ts.done(coll_alltoallv_impl(c, b, counts_dev, send_cap, recv_cap, dt, algo, stream, recv_counts_dev));
}

coll_status_t coll_moe_dispatch(sim_comm_t c, const void* const* x, const int32_t* const* topk_idx, size_t tokens,
                                int k, size_t hidden, int experts, coll_dtype_t dt, void* const* recv,
                                size_t recv_cap_rows, int32_t* const* route_pos, long long* expert_counts_dev,
                                long long* recv_counts_dev, coll_stream_t stream) {
    TraceScope ts(c, "moe_dispatch", tokens, int(dt), -1, -1, -1, stream);
    return ts.done(coll_moe_dispatch_impl(c, x, topk_idx, tokens, k, hidden, experts, dt, recv, recv_cap_rows,
                                          route_pos, expert_counts_dev, recv_counts_dev, stream));
}

coll_status_t coll_moe_combine(sim_comm_t c, const void* const* y, size_t y_rows, const int32_t* const* topk_idx,
                               const int32_t* const* route_pos, const float* const* topk_weight,
                               const void* const* residual, size_t tokens, int k, size_t hidden, int experts,
                               coll_dtype_t dt, void* const* out, coll_stream_t stream) {
    TraceScope ts(c, "moe_combine", tokens, int(dt), -1, -1, -1, stream);
    return ts.done(coll_moe_combine_impl(c, y, y_rows, topk_idx, route_pos, topk_weight, residual, tokens, k, hidden,
                                         experts, dt, out, stream));
}

}  // extern "C"
