// Tree executor: the single and the double binary tree AllReduce.
//
// "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All"
// (charlestar.github.io/2026/08/20/gpu-collective-communication), "Tree AllReduce 为什么更适合延迟敏感区间":
// reduce up a tree to its root, then broadcast down the same tree, in a number of rounds that grows
// with log p. "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives),
// §2.4: the double binary tree runs two complementary trees at once, drawn as tree A = 0 -> {1, 2},
// 1 -> {3, 4}, 2 -> {5, 6} and tree B with rank p-1-m where tree A has rank m.
// Readings (ours): a tree is the heap numbering of positions m = 0..p-1 (children 2m+1, 2m+2); tree A
// holds rank m at position m, tree B rank p-1-m. A position's partial is (own input ⊕ left child's
// partial) ⊕ right child's partial, in fp32 for fp32/bf16 data; a leaf's partial is its input, read
// in place by the parent. The root scales for AVG, rounds once and writes its own output; every
// other position then copies its parent's output. The double tree reduces elements [0, half) on
// tree A and [half, n) on tree B, half = ceil(n/2).
//
// Execution: a tree's range is cut into chunks (the pipelining unit) and a chunk into tiles; every
// (step, tree, chunk, position, tile) is a CTA task. Steps are the reduce levels, deepest first,
// then the broadcast levels, root side first; tasks are claimed from a counter in step order, so a
// task's predecessors (its children's chunk, or its parent's) were claimed earlier by running CTAs
// and every bounded wait ends. A finished task counts itself into its (phase, tree, position,
// chunk) flag, tagged with the call's epoch.
#include "common.cuh"

namespace simcomm {

constexpr int kTreeThreads = 256;
constexpr int kTreeUnroll = 2;

template <int DT>
__device__ __forceinline__ void tree_load_pack(const void* base, bool part, size_t g,
                                               typename Pack16<DT>::A (&x)[Pack16<DT>::L]) {
    if constexpr (DT == COLL_BF16) {
        if (part) {  // a bf16 pack's fp32 partials span two 16-byte words
            const uint4 lo = ld_cg_v4(static_cast<const uint4*>(base) + 2 * g);
            const uint4 hi = ld_cg_v4(static_cast<const uint4*>(base) + 2 * g + 1);
            const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int l = 0; l < 8; ++l) x[l] = __uint_as_float(w[l]);
            return;
        }
    }
    Pack16<DT>::unpack(ld_cg_v4(static_cast<const uint4*>(base) + g), x);
}

template <int DT>
__device__ __forceinline__ typename Elem<DT>::A tree_load_one(const void* base, bool part, size_t e) {
    if (part) {
        if constexpr (DT == COLL_INT32) return int32_t(ld_cg_u32(static_cast<const int32_t*>(base) + e));
        else return __uint_as_float(ld_cg_u32(static_cast<const float*>(base) + e));
    }
    if constexpr (DT == COLL_BF16) return bf16_bits_to_float(ld_cg_u16(static_cast<const uint16_t*>(base) + e));
    else if constexpr (DT == COLL_FP32) return __uint_as_float(ld_cg_u32(static_cast<const float*>(base) + e));
    else return int32_t(ld_cg_u32(static_cast<const int32_t*>(base) + e));
}

// dst = (own ⊕ kid0) ⊕ kid1 over count elements (nk = 0, 1 or 2 kids; a kid is a partial in the
// accumulator type or a leaf's raw input). A final result is scaled for AVG and rounded to the
// element type, otherwise stored as a partial.
template <int DT, int OP, bool SCALE>
__device__ __forceinline__ void tree_fold(const void* own, const void* k0, bool p0, const void* k1, bool p1, int nk,
                                          void* dst, bool final_out, size_t count, float scale, bool vec) {
    using PK = Pack16<DT>;
    using A = typename PK::A;
    constexpr int L = PK::L;
    size_t done = 0;
    if (vec) {
        const size_t ng = count / L;
        for (size_t g0 = threadIdx.x; g0 < ng; g0 += size_t(kTreeThreads) * kTreeUnroll) {
            A xo[kTreeUnroll][L], xa[kTreeUnroll][L], xb[kTreeUnroll][L];
#pragma unroll
            for (int u = 0; u < kTreeUnroll; ++u) {
                const size_t g = g0 + size_t(u) * kTreeThreads;
                if (g < ng) {
                    tree_load_pack<DT>(own, false, g, xo[u]);
                    if (nk > 0) tree_load_pack<DT>(k0, p0, g, xa[u]);
                    if (nk > 1) tree_load_pack<DT>(k1, p1, g, xb[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kTreeUnroll; ++u) {
                const size_t g = g0 + size_t(u) * kTreeThreads;
                if (g >= ng) continue;
                if (nk > 0) fold_into<DT, OP, A, L>(xo[u], xa[u]);
                if (nk > 1) fold_into<DT, OP, A, L>(xo[u], xb[u]);
                if (final_out) {
                    if constexpr (SCALE) {
#pragma unroll
                        for (int l = 0; l < L; ++l) xo[u][l] = xo[u][l] * scale;
                    }
                    st_v4(static_cast<uint4*>(dst) + g, PK::pack(xo[u]));
                } else if constexpr (DT == COLL_BF16) {
                    st_v4(static_cast<uint4*>(dst) + 2 * g,
                          make_uint4(__float_as_uint(xo[u][0]), __float_as_uint(xo[u][1]), __float_as_uint(xo[u][2]),
                                     __float_as_uint(xo[u][3])));
                    st_v4(static_cast<uint4*>(dst) + 2 * g + 1,
                          make_uint4(__float_as_uint(xo[u][4]), __float_as_uint(xo[u][5]), __float_as_uint(xo[u][6]),
                                     __float_as_uint(xo[u][7])));
                } else {
                    st_v4(static_cast<uint4*>(dst) + g, PK::pack(xo[u]));
                }
            }
        }
        done = ng * L;
    }
    for (size_t e = done + threadIdx.x; e < count; e += kTreeThreads) {
        A x = tree_load_one<DT>(own, false, e);
        for (int k = 0; k < nk; ++k) {
            const A y = tree_load_one<DT>(k == 0 ? k0 : k1, k == 0 ? p0 : p1, e);
            if constexpr (DT == COLL_INT32) x = op_i<OP>(x, y);
            else x = op_f<OP>(x, y);
        }
        if (final_out) {
            if constexpr (SCALE) x = x * scale;
            store_elem<DT>(dst, e, x);
        } else {
            static_cast<A*>(dst)[e] = x;
        }
    }
}

__device__ __forceinline__ void tree_copy(const char* s, char* d, size_t bytes) {
    if ((((reinterpret_cast<uintptr_t>(s) | reinterpret_cast<uintptr_t>(d) | bytes) & 15u) == 0)) {
        const size_t nv = bytes / 16;
        for (size_t i0 = threadIdx.x; i0 < nv; i0 += size_t(kTreeThreads) * 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + u * kTreeThreads < nv) v[u] = ld_cg_v4(reinterpret_cast<const uint4*>(s) + i0 + u * kTreeThreads);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + u * kTreeThreads < nv) st_v4(reinterpret_cast<uint4*>(d) + i0 + u * kTreeThreads, v[u]);
        }
    } else {
        for (size_t b = 2 * size_t(threadIdx.x); b < bytes; b += 2 * kTreeThreads)
            *reinterpret_cast<uint16_t*>(d + b) = ld_cg_u16(s + b);
    }
}

__device__ __forceinline__ unsigned long long* tree_flag(const TreeArgs& a, int phase, int b, int m, uint32_t c) {
    return a.flags + ((size_t(phase) * 2 + b) * a.p + m) * a.nchmax + c;
}

template <int DT, int OP, bool SCALE>
__global__ void __launch_bounds__(kTreeThreads, 2) k_tree(const __grid_constant__ TreeArgs a) {
    __shared__ uint32_t s_task;
    __shared__ int s_ok;
    const int p = a.p;
    const size_t d = size_t(Elem<DT>::kBytes);
    constexpr size_t kAcc = sizeof(typename Elem<DT>::A);
    const unsigned long long want = ((unsigned long long)a.epoch << 32) | a.ntile;
    if (threadIdx.x == 0) s_ok = !status_failed(a.ctl);
    __syncthreads();
    const uint32_t total = s_ok ? a.start[a.nsteps] : 0u;
    __syncthreads();
    while (total) {
        if (threadIdx.x == 0) s_task = status_failed(a.ctl) ? total : atomicAdd(&a.st->task_ctr, 1u);
        __syncthreads();
        const uint32_t task = s_task;
        if (task >= total) break;
        uint32_t g = 0;
        while (task >= a.start[g + 1]) ++g;
        // decode (tree, chunk, position, tile) inside step g
        uint32_t rem = task - a.start[g];
        const uint32_t per_chunk = a.step_count[g] * a.ntile;
        int b = 0;
        if (a.ntrees == 2 && rem >= a.nch[0] * per_chunk) {
            rem -= a.nch[0] * per_chunk;
            b = 1;
        }
        const uint32_t c = rem / per_chunk;
        rem -= c * per_chunk;
        const int m = int(a.step_first[g] + rem / a.ntile);
        const uint32_t t = rem % a.ntile;
        const bool reduce = a.step_kind[g] == 0;
        auto rank_at = [&](int pos) { return b == 0 ? pos : p - 1 - pos; };
        auto internal = [&](int pos) { return 2 * pos + 1 < p; };

        // wait for the predecessors' chunk: the internal children (reduce) or the parent (broadcast)
        if (threadIdx.x == 0) {
            int ok = 1;
            if (reduce) {
                for (int k = 2 * m + 1; ok && k <= 2 * m + 2 && k < p; ++k)
                    if (internal(k)) ok = wait_flag(a.ctl, tree_flag(a, 0, b, k, c), want, a.timeout_ns);
            } else {
                const int q = (m - 1) / 2;
                ok = wait_flag(a.ctl, tree_flag(a, q == 0 ? 0 : 1, b, q, c), want, a.timeout_ns);
            }
            s_ok = ok;
        }
        __syncthreads();
        if (!s_ok) break;

        const size_t rlo = b == 0 ? 0 : a.half, rhi = b == 0 ? a.half : a.n;
        const size_t clo = min(rlo + size_t(c) * a.chunk, rhi), chi = min(clo + a.chunk, rhi);
        const size_t lo = min(clo + size_t(t) * a.tile, chi), hi = min(lo + a.tile, chi);
        if (hi > lo) {
            if (reduce) {
                const void* kid[2] = {nullptr, nullptr};
                bool part[2] = {false, false};
                int nk = 0;
                for (int k = 2 * m + 1; k <= 2 * m + 2 && k < p; ++k, ++nk) {
                    part[nk] = internal(k);
                    kid[nk] = part[nk] ? static_cast<const void*>(a.stage + size_t(rank_at(k)) * a.stage_stride + lo * kAcc)
                                       : static_cast<const void*>(static_cast<const char*>(a.ptrs.send[rank_at(k)]) + lo * d);
                }
                const void* own = static_cast<const char*>(a.ptrs.send[rank_at(m)]) + lo * d;
                void* dst = (m == 0) ? static_cast<void*>(static_cast<char*>(a.ptrs.recv[rank_at(0)]) + lo * d)
                                     : static_cast<void*>(a.stage + size_t(rank_at(m)) * a.stage_stride + lo * kAcc);
                tree_fold<DT, OP, SCALE>(own, kid[0], part[0], kid[1], part[1], nk, dst, m == 0, hi - lo, a.scale,
                                         a.vec != 0);
            } else {
                const int q = (m - 1) / 2;
                tree_copy(static_cast<const char*>(a.ptrs.recv[rank_at(q)]) + lo * d,
                          static_cast<char*>(a.ptrs.recv[rank_at(m)]) + lo * d, (hi - lo) * d);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0 && rank_at(m) != a.skip_rank)  // fault injection silences one rank
            signal_chunk(a.ctl, tree_flag(a, reduce ? 0 : 1, b, m, c), a.epoch);
    }
    // Leave: the last CTA out resets the task counter for the next call.
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

template <int DT>
static cudaError_t launch_tree_dt(const TreeArgs& a, int op, int ctas, cudaStream_t s) {
    switch (op) {
        case COLL_SUM: k_tree<DT, COLL_SUM, false><<<ctas, kTreeThreads, 0, s>>>(a); break;
        case COLL_MIN: k_tree<DT, COLL_MIN, false><<<ctas, kTreeThreads, 0, s>>>(a); break;
        case COLL_MAX: k_tree<DT, COLL_MAX, false><<<ctas, kTreeThreads, 0, s>>>(a); break;
        case COLL_AVG:
            if constexpr (DT == COLL_INT32) return cudaErrorInvalidValue;
            else k_tree<DT, COLL_SUM, true><<<ctas, kTreeThreads, 0, s>>>(a);
            break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_tree(const TreeArgs& a, int dtype, int op, int ctas, cudaStream_t s) {
    switch (dtype) {
        case COLL_INT32: return launch_tree_dt<COLL_INT32>(a, op, ctas, s);
        case COLL_FP32: return launch_tree_dt<COLL_FP32>(a, op, ctas, s);
        case COLL_BF16: return launch_tree_dt<COLL_BF16>(a, op, ctas, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace simcomm
