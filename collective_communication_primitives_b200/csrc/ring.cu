// Ring executor: the chunk-pipelined ring schedules, run by one persistent kernel.
//
// Schedule ("集合通信：原语、算法、NCCL 实现与拓扑映射", llm-infra-atlas.github.io/hpc/04_collectives,
// §2.2 ring all-reduce; chunking and pipelining §3.5): the ranks form the ring r0 -> r1 -> ... ->
// r_{p-1} -> r0 and every buffer is cut into p segments.
//   reduce-scatter step s = 1..p-1: rank r receives segment k = (r-1-s) mod p from rank r-1 and
//     stores received ⊕ own; at step p-1, k = r and the result is final (scaled for AVG, rounded);
//   all-gather step s = 1..p-1: rank r copies segment k = (r-s) mod p from rank r-1.
// (The page's p = 4 trace is garbled; this is the reading under which rank r ends up owning block
// r, as ReduceScatter requires.) Partials of bf16 data travel in fp32.
// Other schedules on the same executor (our reading, the pages give rings only for the above):
//   Reduce: chain root+1 -> ... -> root;  Broadcast: chain root -> ... -> root-1;
//   All-to-All(v): p shift steps, at step s rank r sends its block for rank (r+s) mod p there.
//
// Execution: every (step, chunk, rank) is a task. CTAs claim tasks from a counter in step-major
// order, so a task's predecessor (step-1, chunk, rank-1) was claimed earlier by a CTA that is
// running; waiting for it therefore always ends. A finished task release-stores the call's epoch
// into its flag; its successor acquire-loads that flag with a bounded wait. One chunk is the
// pipelining unit: chunk c of step s+1 starts as soon as chunk c of step s is done on the
// predecessor, while other chunks are still in earlier steps.
#include "a2av.cuh"
#include "common.cuh"

namespace simcomm {

constexpr int kRingThreads = 256;
constexpr int kHopUnroll = 4;

// ---- hop bodies (run by the whole CTA) ------------------------------------------------------------

template <int DT>
__device__ __forceinline__ typename Elem<DT>::A load_elem_cg(const void* base, size_t e) {
    if constexpr (DT == COLL_BF16) return bf16_bits_to_float(ld_cg_u16(static_cast<const uint16_t*>(base) + e));
    else if constexpr (DT == COLL_FP32) return __uint_as_float(ld_cg_u32(static_cast<const float*>(base) + e));
    else return int32_t(ld_cg_u32(static_cast<const int32_t*>(base) + e));
}

// dst[e] = wire[e] ⊕ own[e] for e < count. wire is a partial (accumulator type, fp32 for bf16) or,
// on a chain's first hop, the predecessor's raw input (element type). The final hop scales for AVG
// and rounds to the element type; other hops store a partial.
template <int DT, int OP, bool SCALE>
__device__ __forceinline__ void hop_reduce(const void* wire, bool wire_partial, const void* own, void* dst,
                                           bool final_out, size_t count, float scale, bool vec) {
    using PK = Pack16<DT>;
    using A = typename PK::A;
    constexpr int L = PK::L;
    constexpr bool kWide = (DT == COLL_BF16);  // partial pack is two 16-byte words
    size_t done = 0;
    if (vec) {
        const size_t ng = count / L;
        for (size_t g0 = threadIdx.x; g0 < ng; g0 += size_t(kRingThreads) * kHopUnroll) {
            uint4 wv[kHopUnroll][2], ov[kHopUnroll];
#pragma unroll
            for (int u = 0; u < kHopUnroll; ++u) {
                const size_t g = g0 + size_t(u) * kRingThreads;
                if (g < ng) {
                    ov[u] = ld_cg_v4(static_cast<const uint4*>(own) + g);
                    if (kWide && wire_partial) {
                        wv[u][0] = ld_cg_v4(static_cast<const uint4*>(wire) + 2 * g);
                        wv[u][1] = ld_cg_v4(static_cast<const uint4*>(wire) + 2 * g + 1);
                    } else {
                        wv[u][0] = ld_cg_v4(static_cast<const uint4*>(wire) + g);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kHopUnroll; ++u) {
                const size_t g = g0 + size_t(u) * kRingThreads;
                if (g >= ng) continue;
                A w[L], o[L];
                bool unpacked = false;
                if constexpr (kWide) {
                    if (wire_partial) {
                        const uint32_t ws[8] = {wv[u][0].x, wv[u][0].y, wv[u][0].z, wv[u][0].w,
                                                wv[u][1].x, wv[u][1].y, wv[u][1].z, wv[u][1].w};
#pragma unroll
                        for (int l = 0; l < 8; ++l) w[l] = __uint_as_float(ws[l]);
                        unpacked = true;
                    }
                }
                if (!unpacked) PK::unpack(wv[u][0], w);
                PK::unpack(ov[u], o);
                fold_into<DT, OP, A, L>(w, o);  // received ⊕ own: the received partial comes first
                if (final_out) {
                    if constexpr (SCALE) {
#pragma unroll
                        for (int l = 0; l < L; ++l) w[l] = w[l] * scale;
                    }
                    st_v4(static_cast<uint4*>(dst) + g, PK::pack(w));
                } else {
                    if constexpr (kWide) {
                        st_v4(static_cast<uint4*>(dst) + 2 * g,
                              make_uint4(__float_as_uint(w[0]), __float_as_uint(w[1]), __float_as_uint(w[2]),
                                         __float_as_uint(w[3])));
                        st_v4(static_cast<uint4*>(dst) + 2 * g + 1,
                              make_uint4(__float_as_uint(w[4]), __float_as_uint(w[5]), __float_as_uint(w[6]),
                                         __float_as_uint(w[7])));
                    } else {
                        st_v4(static_cast<uint4*>(dst) + g, PK::pack(w));
                    }
                }
            }
        }
        done = ng * L;
    }
    for (size_t e = done + threadIdx.x; e < count; e += kRingThreads) {
        A w;
        if (wire_partial) {
            if constexpr (DT == COLL_INT32) w = int32_t(ld_cg_u32(static_cast<const int32_t*>(wire) + e));
            else w = __uint_as_float(ld_cg_u32(static_cast<const float*>(wire) + e));
        } else {
            w = load_elem_cg<DT>(wire, e);
        }
        const A o = load_elem_cg<DT>(own, e);
        if constexpr (DT == COLL_INT32) w = op_i<OP>(w, o);
        else w = op_f<OP>(w, o);
        if (final_out) {
            if constexpr (SCALE) w = w * scale;
            store_elem<DT>(dst, e, w);
        } else {
            static_cast<A*>(dst)[e] = w;
        }
    }
}

// dst[0, bytes) = src[0, bytes); 16-byte accesses where source and destination agree modulo 16,
// 2-byte accesses otherwise (all element sizes are 2 or 4 bytes).
__device__ __forceinline__ void hop_copy(const void* src, void* dst, size_t bytes) {
    const char* s = static_cast<const char*>(src);
    char* d = static_cast<char*>(dst);
    size_t head = bytes, body = 0;
    if (((reinterpret_cast<uintptr_t>(s) ^ reinterpret_cast<uintptr_t>(d)) & 15u) == 0) {
        head = (16 - (reinterpret_cast<uintptr_t>(s) & 15u)) & 15u;
        if (head > bytes) head = bytes;
        body = (bytes - head) & ~size_t(15);
    }
    for (size_t b = 2 * size_t(threadIdx.x); b < head; b += 2 * kRingThreads)
        *reinterpret_cast<uint16_t*>(d + b) = ld_cg_u16(s + b);
    const uint4* vs = reinterpret_cast<const uint4*>(s + head);
    uint4* vd = reinterpret_cast<uint4*>(d + head);
    const size_t nv = body / 16;
    for (size_t v0 = threadIdx.x; v0 < nv; v0 += size_t(kRingThreads) * kHopUnroll) {
        uint4 t[kHopUnroll];
#pragma unroll
        for (int u = 0; u < kHopUnroll; ++u) {
            const size_t v = v0 + size_t(u) * kRingThreads;
            if (v < nv) t[u] = ld_cg_v4(vs + v);
        }
#pragma unroll
        for (int u = 0; u < kHopUnroll; ++u) {
            const size_t v = v0 + size_t(u) * kRingThreads;
            if (v < nv) st_v4(vd + v, t[u]);
        }
    }
    for (size_t b = head + body + 2 * size_t(threadIdx.x); b < bytes; b += 2 * kRingThreads)
        *reinterpret_cast<uint16_t*>(d + b) = ld_cg_u16(s + b);
}

// ---- the executor ------------------------------------------------------------------------------

struct Task {
    bool wait;         // wait for the predecessor's flag before working
    uint32_t pred;     // its flag index
};

__device__ __forceinline__ int md(int a, int p) { return ((a % p) + p) % p; }

template <int DT, int OP, bool SCALE>
__global__ void __launch_bounds__(kRingThreads) k_ring(const __grid_constant__ RingArgs a) {
    extern __shared__ __align__(16) unsigned char dyn_smem[];
    __shared__ uint32_t s_task;
    __shared__ int s_ok;
    __shared__ uint32_t s_nch;

    const int p = a.p;
    const size_t d = size_t(Elem<DT>::kBytes);
    constexpr size_t kAcc = sizeof(typename Elem<DT>::A);
    long long* sd = reinterpret_cast<long long*>(dyn_smem);
    long long* rd = sd + p * p;

    // One thread decides whether this CTA runs, so the decision is uniform across the CTA.
    if (threadIdx.x == 0) s_ok = !status_failed(a.ctl);
    __syncthreads();
    bool run = s_ok;
    __syncthreads();
    uint32_t nch = a.nch;
    if (a.kind == RING_ALLTOALLV && run) {
        if (threadIdx.x < 32) {
            const A2avPlan plan = a2av_plan_warp(a.counts, p, a.send_cap, a.recv_cap, sd, rd, a.recv_counts_out, a.ctl);
            if (threadIdx.x == 0) {
                s_ok = plan.ok;
                s_nch = plan.max_count > 0 ? uint32_t((size_t(plan.max_count) + a.chunk - 1) / a.chunk) : 0u;
            }
        }
        __syncthreads();
        run = s_ok;
        nch = s_nch;
    }
    const uint32_t rps = a.ranks_per_step;
    const uint32_t per_step = rps * nch;
    const uint32_t total = run ? a.nsteps * per_step : 0u;

    while (total) {
        if (threadIdx.x == 0) s_task = status_failed(a.ctl) ? total : atomicAdd(&a.st->task_ctr, 1u);
        __syncthreads();
        const uint32_t t = s_task;
        if (t >= total) break;
        const uint32_t g = t / per_step;
        const uint32_t rem = t - g * per_step;
        const uint32_t c = rem / rps;
        const int r = int(rem - c * rps);
        const uint32_t my_flag = (g * rps + uint32_t(r)) * nch + c;
        Task tk{false, 0};
        int signal_rank = r;

        switch (a.kind) {
            case RING_ALLREDUCE:
            case RING_REDUCE_SCATTER:
                if (g >= 1) tk = Task{true, ((g - 1) * rps + uint32_t(md(r - 1, p))) * nch + c};
                break;
            case RING_ALLGATHER:
                if (g >= 2) tk = Task{true, ((g - 1) * rps + uint32_t(md(r - 1, p))) * nch + c};
                break;
            case RING_REDUCE:
                signal_rank = md(a.root + 2 + int(g), p);
                if (g >= 1) tk = Task{true, (g - 1) * nch + c};
                break;
            case RING_BCAST:
                signal_rank = md(a.root + int(g), p);
                if (g >= 2) tk = Task{true, (g - 1) * nch + c};
                break;
            default:
                break;
        }
        if (tk.wait) {
            if (threadIdx.x == 0) s_ok = wait_flag(a.ctl, a.flags + tk.pred, a.epoch, a.timeout_ns);
            __syncthreads();
            if (!s_ok) break;
        }

        switch (a.kind) {
            case RING_ALLREDUCE:
            case RING_REDUCE_SCATTER: {
                const int w = md(r - 1, p);
                const bool rs_phase = (a.kind == RING_REDUCE_SCATTER) || g < uint32_t(p - 1);
                const int s = rs_phase ? int(g) + 1 : int(g) - (p - 1) + 1;
                const int k = rs_phase ? md(r - 1 - s, p) : md(r - s, p);
                const size_t sb = min(size_t(k) * a.seg, a.n), se = min(sb + a.seg, a.n);
                const size_t lo = min(sb + size_t(c) * a.chunk, se), hi = min(lo + a.chunk, se);
                if (hi > lo) {
                    if (rs_phase) {
                        const bool first = (s == 1), last = (s == p - 1);
                        const void* wire = first ? static_cast<const void*>(static_cast<const char*>(a.ptrs.send[w]) + lo * d)
                                                 : static_cast<const void*>(a.stage + size_t(w) * a.stage_stride + lo * kAcc);
                        const void* own = static_cast<const char*>(a.ptrs.send[r]) + lo * d;
                        void* dst;
                        if (!last) dst = a.stage + size_t(r) * a.stage_stride + lo * kAcc;
                        else if (a.kind == RING_ALLREDUCE) dst = static_cast<char*>(a.ptrs.recv[r]) + lo * d;
                        else dst = static_cast<char*>(a.ptrs.recv[r]) + (lo - sb) * d;
                        hop_reduce<DT, OP, SCALE>(wire, !first, own, dst, last, hi - lo, a.scale, a.vec != 0);
                    } else {
                        hop_copy(static_cast<const char*>(a.ptrs.recv[w]) + lo * d,
                                 static_cast<char*>(a.ptrs.recv[r]) + lo * d, (hi - lo) * d);
                    }
                }
                break;
            }
            case RING_ALLGATHER: {
                // g = 0: the own shard into the own output; g = s >= 1: segment (r-s) mod p from r-1
                const int k = (g == 0) ? r : md(r - int(g), p);
                const size_t lo = min(size_t(c) * a.chunk, a.seg), hi = min(lo + a.chunk, a.seg);
                if (hi > lo) {
                    char* dst = static_cast<char*>(a.ptrs.recv[r]) + (size_t(k) * a.seg + lo) * d;
                    const char* src;
                    if (g == 0) src = static_cast<const char*>(a.ptrs.send[r]) + lo * d;
                    else if (g == 1) src = static_cast<const char*>(a.ptrs.send[md(r - 1, p)]) + lo * d;
                    else src = static_cast<const char*>(a.ptrs.recv[md(r - 1, p)]) + (size_t(k) * a.seg + lo) * d;
                    if (src != dst) hop_copy(src, dst, (hi - lo) * d);
                }
                break;
            }
            case RING_REDUCE: {
                // hop h = g+1 at rank q = root+1+h, its predecessor w = q-1
                const int h = int(g) + 1;
                const int q = md(a.root + 1 + h, p), w = md(q - 1, p);
                const size_t lo = min(size_t(c) * a.chunk, a.n), hi = min(lo + a.chunk, a.n);
                if (hi > lo) {
                    const bool first = (h == 1), last = (h == p - 1);
                    const void* wire = first ? static_cast<const void*>(static_cast<const char*>(a.ptrs.send[w]) + lo * d)
                                             : static_cast<const void*>(a.stage + size_t(w) * a.stage_stride + lo * kAcc);
                    const void* own = static_cast<const char*>(a.ptrs.send[q]) + lo * d;
                    void* dst = last ? static_cast<void*>(static_cast<char*>(a.ptrs.recv[a.root]) + lo * d)
                                     : static_cast<void*>(a.stage + size_t(q) * a.stage_stride + lo * kAcc);
                    hop_reduce<DT, OP, SCALE>(wire, !first, own, dst, last, hi - lo, a.scale, a.vec != 0);
                }
                break;
            }
            case RING_BCAST: {
                // hop 0: the root's own output; hop h >= 1: rank root+h copies from its predecessor
                const int q = md(a.root + int(g), p);
                const size_t lo = min(size_t(c) * a.chunk, a.n), hi = min(lo + a.chunk, a.n);
                if (hi > lo) {
                    const char* src = (g <= 1) ? static_cast<const char*>(a.ptrs.send[a.root])
                                               : static_cast<const char*>(a.ptrs.recv[md(q - 1, p)]);
                    char* dst = static_cast<char*>(a.ptrs.recv[q]);
                    if (src + lo * d != dst + lo * d) hop_copy(src + lo * d, dst + lo * d, (hi - lo) * d);
                }
                break;
            }
            case RING_ALLTOALL:
            case RING_ALLTOALLV: {
                const int j = md(r + int(g), p);
                size_t len, soff, roff;
                if (a.kind == RING_ALLTOALL) {
                    len = a.seg; soff = size_t(j) * a.seg; roff = size_t(r) * a.seg;
                } else {
                    len = size_t(a.counts[r * p + j]); soff = size_t(sd[r * p + j]); roff = size_t(rd[r * p + j]);
                }
                const size_t lo = min(size_t(c) * a.chunk, len), hi = min(lo + a.chunk, len);
                if (hi > lo)
                    hop_copy(static_cast<const char*>(a.ptrs.send[r]) + (soff + lo) * d,
                             static_cast<char*>(a.ptrs.recv[j]) + (roff + lo) * d, (hi - lo) * d);
                break;
            }
            default:
                break;
        }

        __syncthreads();
        // The All-to-All schedules have no dependent steps and no flags.
        const bool has_flags = (a.kind != RING_ALLTOALL && a.kind != RING_ALLTOALLV);
        if (threadIdx.x == 0 && has_flags && signal_rank != a.skip_rank) {
            __threadfence();
            st_release_gpu(a.flags + my_flag, a.epoch);
        }
    }

    // Leave: the last CTA out resets the task counter for the next call on this communicator.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&a.st->done_ctr, 1u) == gridDim.x - 1) {
            a.st->task_ctr = 0;
            a.st->done_ctr = 0;
            __threadfence();
        }
    }
}

template <int DT, int OP, bool SCALE>
static cudaError_t launch_ring_typed(const RingArgs& a, int ctas, cudaStream_t s) {
    const size_t smem = (a.kind == RING_ALLTOALLV) ? 2 * size_t(a.p) * a.p * sizeof(long long) : 0;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_ring<DT, OP, SCALE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(2 * size_t(kMaxRanks) * kMaxRanks * sizeof(long long)));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    k_ring<DT, OP, SCALE><<<ctas, kRingThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int DT>
static cudaError_t launch_ring_dt(const RingArgs& a, int op, int ctas, cudaStream_t s) {
    switch (op) {
        case COLL_SUM: return launch_ring_typed<DT, COLL_SUM, false>(a, ctas, s);
        case COLL_MIN: return launch_ring_typed<DT, COLL_MIN, false>(a, ctas, s);
        case COLL_MAX: return launch_ring_typed<DT, COLL_MAX, false>(a, ctas, s);
        case COLL_AVG:
            if constexpr (DT == COLL_INT32) return cudaErrorInvalidValue;
            else return launch_ring_typed<DT, COLL_SUM, true>(a, ctas, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_ring(const RingArgs& a, int dtype, int op, int ctas, cudaStream_t s) {
    switch (dtype) {
        case COLL_INT32: return launch_ring_dt<COLL_INT32>(a, op, ctas, s);
        case COLL_FP32: return launch_ring_dt<COLL_FP32>(a, op, ctas, s);
        case COLL_BF16: return launch_ring_dt<COLL_BF16>(a, op, ctas, s);
        default: return cudaErrorInvalidValue;
    }
}

int ring_max_ctas(int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_ring<COLL_FP32, COLL_SUM, false>, kRingThreads,
                                                      0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    return num_sms * per_sm;
}

}  // namespace simcomm
