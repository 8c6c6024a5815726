// Direct fused reduction: AllReduce, Reduce and ReduceScatter in one pass.
//
// Each thread takes a 32-byte (or 16-byte) position i of the reduced range, loads that position from all p
// ranks' inputs (all loads issued before the first add), folds them in rank order in fp32 (bf16 is
// widened; int32 wraps), scales by 1/p for AVG, rounds once, and stores the result to every owner:
// all p outputs for AllReduce, the root's output for Reduce, the owner's shard for ReduceScatter.
// Every input byte is read once and every output byte written once, the minimum HBM traffic of a
// collective whose ranks share one memory.
//
// Semantics ("集合通信：原语、算法、NCCL 实现与拓扑映射", llm-infra-atlas.github.io/hpc/04_collectives):
//   §1.3 Reduce:        out_root[i] = ⊕_r in_r[i]
//   §1.4 AllReduce:     out_r[i]    = ⊕_r' in_r'[i] for every r
//   §1.5 ReduceScatter: out_r[k]    = ⊕_q in_q[r·m + k], m = n/p
#include <algorithm>

#include "common.cuh"

namespace simcomm {

constexpr int kDirThreads = 256;
constexpr int kDirUnroll = 2;  // 16-byte positions per thread per iteration
constexpr int kDirGroup = 8;   // ranks loaded together when p is only known at run time

// ---- element-wise path (unaligned buffers and the ragged tail) -----------------------------------

// Reduce input element e (0 <= e < n) and store it to its owner(s).
template <int DT, int OP, bool SCALE>
__device__ __forceinline__ void reduce_one_element(const DirectReduceArgs& a, int p, size_t e) {
    using A = typename Elem<DT>::A;
    A acc = load_elem<DT>(a.ptrs.send[0], e);
    for (int q = 1; q < p; ++q) {
        A x = load_elem<DT>(a.ptrs.send[q], e);
        if constexpr (DT == COLL_INT32) acc = op_i<OP>(acc, x);
        else acc = op_f<OP>(acc, x);
    }
    if constexpr (SCALE) acc = acc * a.scale;
    if (a.mode == MODE_ALLREDUCE) {
        for (int r = 0; r < p; ++r) store_elem<DT>(a.ptrs.recv[r], e, acc);
    } else if (a.mode == MODE_REDUCE) {
        store_elem<DT>(a.ptrs.recv[a.root], e, acc);
    } else {
        const size_t owner = e / a.seg;
        store_elem<DT>(a.ptrs.recv[owner], e - owner * a.seg, acc);
    }
}

template <int DT, int OP, bool SCALE>
__global__ void __launch_bounds__(kDirThreads) k_direct_scalar(const __grid_constant__ DirectReduceArgs a) {
    __shared__ int s_stop;
    if (threadIdx.x == 0) s_stop = status_failed(a.ctl);
    __syncthreads();
    if (s_stop) return;
    const size_t stride = size_t(gridDim.x) * kDirThreads;
    for (size_t e = size_t(blockIdx.x) * kDirThreads + threadIdx.x; e < a.n; e += stride)
        reduce_one_element<DT, OP, SCALE>(a, a.p, e);
}

// ---- 16-byte path ------------------------------------------------------------------------------

// P > 0: p is a compile-time constant and all p loads of a position are in flight together.
// P == 0: p is read at run time and ranks are loaded kDirGroup at a time.
// W: 32-bit words per pack (4: 16-byte accesses, 8: 32-byte accesses).
template <int DT, int OP, int P, bool SCALE, int W, bool HINT>
__global__ void __launch_bounds__(kDirThreads) k_direct_vec(const __grid_constant__ DirectReduceArgs a) {
    using PK = PackW<DT, W>;
    using A = typename PK::A;
    constexpr int L = PK::L;
    constexpr int G = (P > 0) ? P : kDirGroup;

    __shared__ int s_stop;
    if (threadIdx.x == 0) s_stop = status_failed(a.ctl);
    __syncthreads();
    if (s_stop) return;

    const int p = (P > 0) ? P : a.p;
    const int nseg = (a.mode == MODE_REDUCE_SCATTER) ? p : 1;
    const size_t seg_packs = a.seg / L;
    uint64_t pol = 0;
    if constexpr (HINT) pol = l2_evict_first_policy();
    const size_t step = size_t(gridDim.x) * kDirThreads * kDirUnroll;

    // ReduceScatter segments are spread over blockIdx.y (all of them in parallel when a segment is
    // too short to fill the grid); AllReduce and Reduce have one segment and gridDim.y == 1.
    for (int sg = blockIdx.y; sg < nseg; sg += gridDim.y) {
        const size_t in_base = size_t(sg) * seg_packs;
        for (size_t i0 = size_t(blockIdx.x) * kDirThreads * kDirUnroll + threadIdx.x; i0 < seg_packs; i0 += step) {
            bool ok[kDirUnroll];
#pragma unroll
            for (int u = 0; u < kDirUnroll; ++u) ok[u] = (i0 + size_t(u) * kDirThreads) < seg_packs;

            A acc[kDirUnroll][L];
            for (int q0 = 0; q0 < p; q0 += G) {
                Words<W> v[kDirUnroll][G];
#pragma unroll
                for (int u = 0; u < kDirUnroll; ++u)
#pragma unroll
                    for (int j = 0; j < G; ++j)
                        if (ok[u] && (P > 0 || q0 + j < p))
                            v[u][j] = ld_pack<W, HINT>(static_cast<const Words<W>*>(a.ptrs.send[q0 + j]) +
                                                           in_base + i0 + size_t(u) * kDirThreads, pol);
#pragma unroll
                for (int u = 0; u < kDirUnroll; ++u) {
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        if (!(P > 0 || q0 + j < p)) continue;
                        A x[L];
                        PK::unpack(v[u][j], x);
                        if (q0 + j == 0) {
#pragma unroll
                            for (int l = 0; l < L; ++l) acc[u][l] = x[l];
                        } else {
                            fold_into<DT, OP, A, L>(acc[u], x);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kDirUnroll; ++u) {
                if (!ok[u]) continue;
                if constexpr (SCALE) {
#pragma unroll
                    for (int l = 0; l < L; ++l) acc[u][l] = acc[u][l] * a.scale;
                }
                const Words<W> out = PK::pack(acc[u]);
                const size_t idx = i0 + size_t(u) * kDirThreads;
                if (a.mode == MODE_ALLREDUCE) {
                    if constexpr (P > 0) {
#pragma unroll
                        for (int r = 0; r < P; ++r)
                            st_pack<W, HINT>(static_cast<Words<W>*>(a.ptrs.recv[r]) + in_base + idx, out, pol);
                    } else {
                        for (int r = 0; r < p; ++r)
                            st_pack<W, HINT>(static_cast<Words<W>*>(a.ptrs.recv[r]) + in_base + idx, out, pol);
                    }
                } else if (a.mode == MODE_REDUCE) {
                    st_pack<W, HINT>(static_cast<Words<W>*>(a.ptrs.recv[a.root]) + in_base + idx, out, pol);
                } else {
                    st_pack<W, HINT>(static_cast<Words<W>*>(a.ptrs.recv[sg]) + idx, out, pol);
                }
            }
        }
    }

    // Ragged tail of AllReduce/Reduce (n not a multiple of the pack): the last block, element-wise.
    if (a.mode != MODE_REDUCE_SCATTER && blockIdx.x == gridDim.x - 1 && blockIdx.y == 0) {
        for (size_t e = seg_packs * L + threadIdx.x; e < a.n; e += kDirThreads)
            reduce_one_element<DT, OP, SCALE>(a, p, e);
    }
}

// ---- launch ------------------------------------------------------------------------------------

// Grid of the 16/32-byte path: x covers the packs of one segment (at most max_blocks), y the
// ReduceScatter segments that fit beside it in max_blocks.
static dim3 vec_grid(const DirectReduceArgs& a, size_t packs, int max_blocks) {
    const size_t want = (packs + size_t(kDirThreads) * kDirUnroll - 1) / (size_t(kDirThreads) * kDirUnroll);
    const int gx = int(want < size_t(max_blocks) ? (want ? want : 1) : size_t(max_blocks));
    int gy = 1;
    if (a.mode == MODE_REDUCE_SCATTER) gy = std::max(1, std::min(a.p, max_blocks / gx));
    return dim3(unsigned(gx), unsigned(gy), 1u);
}

template <int DT, int OP, bool SCALE>
static cudaError_t launch_typed(const DirectReduceArgs& a, int num_sms, cudaStream_t s) {
    // ctas_per_sm == 0: one pass, every CTA takes one iteration's worth of positions (the blocks are
    // dispatched in address order as SMs free up)
    const int max_blocks = a.ctas_per_sm > 0 ? num_sms * a.ctas_per_sm : (1 << 30);
    if (!a.vec) {
        const size_t want = (a.n + kDirThreads - 1) / kDirThreads;
        const int grid = int(want < size_t(max_blocks) ? (want ? want : 1) : size_t(max_blocks));
        k_direct_scalar<DT, OP, SCALE><<<grid, kDirThreads, 0, s>>>(a);
        return cudaGetLastError();
    }
    // 32-byte packs when every buffer allows them, else 16-byte packs
    if (a.vec == 2) {
        const dim3 grid = vec_grid(a, a.seg / PackW<DT, 8>::L, max_blocks);
        if (a.l2_hint) {
            switch (a.p) {
                case 2: k_direct_vec<DT, OP, 2, SCALE, 8, true><<<grid, kDirThreads, 0, s>>>(a); break;
                case 4: k_direct_vec<DT, OP, 4, SCALE, 8, true><<<grid, kDirThreads, 0, s>>>(a); break;
                case 8: k_direct_vec<DT, OP, 8, SCALE, 8, true><<<grid, kDirThreads, 0, s>>>(a); break;
                default: k_direct_vec<DT, OP, 0, SCALE, 8, true><<<grid, kDirThreads, 0, s>>>(a); break;
            }
            return cudaGetLastError();
        }
        switch (a.p) {
            case 2: k_direct_vec<DT, OP, 2, SCALE, 8, false><<<grid, kDirThreads, 0, s>>>(a); break;
            case 4: k_direct_vec<DT, OP, 4, SCALE, 8, false><<<grid, kDirThreads, 0, s>>>(a); break;
            case 8: k_direct_vec<DT, OP, 8, SCALE, 8, false><<<grid, kDirThreads, 0, s>>>(a); break;
            default: k_direct_vec<DT, OP, 0, SCALE, 8, false><<<grid, kDirThreads, 0, s>>>(a); break;
        }
        return cudaGetLastError();
    }
    const dim3 grid = vec_grid(a, a.seg / PackW<DT, 4>::L, max_blocks);
    switch (a.p) {
        case 2: k_direct_vec<DT, OP, 2, SCALE, 4, false><<<grid, kDirThreads, 0, s>>>(a); break;
        case 3: k_direct_vec<DT, OP, 3, SCALE, 4, false><<<grid, kDirThreads, 0, s>>>(a); break;
        case 4: k_direct_vec<DT, OP, 4, SCALE, 4, false><<<grid, kDirThreads, 0, s>>>(a); break;
        case 8: k_direct_vec<DT, OP, 8, SCALE, 4, false><<<grid, kDirThreads, 0, s>>>(a); break;
        default: k_direct_vec<DT, OP, 0, SCALE, 4, false><<<grid, kDirThreads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

template <int DT>
static cudaError_t launch_dt(const DirectReduceArgs& a, int op, int num_sms, cudaStream_t s) {
    switch (op) {
        case COLL_SUM: return launch_typed<DT, COLL_SUM, false>(a, num_sms, s);
        case COLL_MIN: return launch_typed<DT, COLL_MIN, false>(a, num_sms, s);
        case COLL_MAX: return launch_typed<DT, COLL_MAX, false>(a, num_sms, s);
        case COLL_AVG:
            if constexpr (DT == COLL_INT32) return cudaErrorInvalidValue;
            else return launch_typed<DT, COLL_SUM, true>(a, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_direct_reduce(const DirectReduceArgs& a, int dtype, int op, int num_sms, cudaStream_t s) {
    switch (dtype) {
        case COLL_INT32: return launch_dt<COLL_INT32>(a, op, num_sms, s);
        case COLL_FP32: return launch_dt<COLL_FP32>(a, op, num_sms, s);
        case COLL_BF16: return launch_dt<COLL_BF16>(a, op, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace simcomm
