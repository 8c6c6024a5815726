// Butterfly executor: the recursive-doubling and recursive halving-doubling AllReduce.
//
// "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives), §2.3 (p a
// power of two):
//   recursive doubling: log2 p steps; at step k every rank exchanges its whole vector with the
//     peer at distance 2^k and reduces, so every rank ends with the reduction (fewest steps,
//     n·log2 p bytes per rank);
//   halving-doubling: a reduce-scatter whose message halves at every step (distances p/2, ..., 1),
//     then an all-gather whose message doubles (distances 1, ..., p/2): 2·log2 p steps, about 2n
//     bytes per rank.
// Reading (the page gives the exchange pattern only): partners combine with the lower rank's data
// first, so both compute the same value; a halving step keeps the half of the rank's block group
// that contains its own block, so rank r ends with the complete block r; partials travel in fp32
// for fp32/bf16 data and are rounded once at the end.
//
// Execution: every (step, rank, tile) is a CTA task, claimed in step order from a counter; a step
// starts when every task of the previous step has finished (a per-step counter the last CTA out
// clears), so a rank can overwrite the buffers the previous step read.
#include "common.cuh"

namespace simcomm {

constexpr int kBflyThreads = 256;
constexpr int kBflyUnroll = 4;

// dst[e] = a[e] ⊕ b[e]; a and b are raw inputs (element type) or partials (accumulator type); a
// final result is scaled for AVG and rounded to the element type, else stored as a partial.
template <int DT, int OP, bool SCALE>
__device__ __forceinline__ void pair_reduce(const void* a, bool a_part, const void* b, bool b_part, void* dst,
                                            bool final_out, size_t count, float scale, bool vec) {
    using PK = Pack16<DT>;
    using A = typename PK::A;
    constexpr int L = PK::L;
    constexpr bool kWide = (DT == COLL_BF16);  // a bf16 pack's partials span two 16-byte words
    auto load_pack = [&](const void* base, bool part, size_t g, A (&x)[L]) {
        if constexpr (kWide) {
            if (part) {
                const uint4 lo = ld_cg_v4(static_cast<const uint4*>(base) + 2 * g);
                const uint4 hi = ld_cg_v4(static_cast<const uint4*>(base) + 2 * g + 1);
                const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int l = 0; l < 8; ++l) x[l] = __uint_as_float(w[l]);
                return;
            }
        }
        PK::unpack(ld_cg_v4(static_cast<const uint4*>(base) + g), x);
    };
    size_t done = 0;
    if (vec) {
        const size_t ng = count / L;
        for (size_t g0 = threadIdx.x; g0 < ng; g0 += size_t(kBflyThreads) * kBflyUnroll) {
            A xa[kBflyUnroll][L], xb[kBflyUnroll][L];
#pragma unroll
            for (int u = 0; u < kBflyUnroll; ++u) {
                const size_t g = g0 + size_t(u) * kBflyThreads;
                if (g < ng) {
                    load_pack(a, a_part, g, xa[u]);
                    load_pack(b, b_part, g, xb[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kBflyUnroll; ++u) {
                const size_t g = g0 + size_t(u) * kBflyThreads;
                if (g >= ng) continue;
                fold_into<DT, OP, A, L>(xa[u], xb[u]);
                if (final_out) {
                    if constexpr (SCALE) {
#pragma unroll
                        for (int l = 0; l < L; ++l) xa[u][l] = xa[u][l] * scale;
                    }
                    st_v4(static_cast<uint4*>(dst) + g, PK::pack(xa[u]));
                } else if constexpr (kWide) {
                    st_v4(static_cast<uint4*>(dst) + 2 * g,
                          make_uint4(__float_as_uint(xa[u][0]), __float_as_uint(xa[u][1]), __float_as_uint(xa[u][2]),
                                     __float_as_uint(xa[u][3])));
                    st_v4(static_cast<uint4*>(dst) + 2 * g + 1,
                          make_uint4(__float_as_uint(xa[u][4]), __float_as_uint(xa[u][5]), __float_as_uint(xa[u][6]),
                                     __float_as_uint(xa[u][7])));
                } else {
                    st_v4(static_cast<uint4*>(dst) + g, PK::pack(xa[u]));
                }
            }
        }
        done = ng * L;
    }
    auto load_one = [&](const void* base, bool part, size_t e) -> A {
        if (part) {
            if constexpr (DT == COLL_INT32) return int32_t(ld_cg_u32(static_cast<const int32_t*>(base) + e));
            else return __uint_as_float(ld_cg_u32(static_cast<const float*>(base) + e));
        }
        if constexpr (DT == COLL_BF16) return bf16_bits_to_float(ld_cg_u16(static_cast<const uint16_t*>(base) + e));
        else if constexpr (DT == COLL_FP32) return __uint_as_float(ld_cg_u32(static_cast<const float*>(base) + e));
        else return int32_t(ld_cg_u32(static_cast<const int32_t*>(base) + e));
    };
    for (size_t e = done + threadIdx.x; e < count; e += kBflyThreads) {
        A x = load_one(a, a_part, e);
        const A y = load_one(b, b_part, e);
        if constexpr (DT == COLL_INT32) x = op_i<OP>(x, y);
        else x = op_f<OP>(x, y);
        if (final_out) {
            if constexpr (SCALE) x = x * scale;
            store_elem<DT>(dst, e, x);
        } else {
            static_cast<A*>(dst)[e] = x;
        }
    }
}

__device__ __forceinline__ void bfly_copy(const char* s, char* d, size_t bytes) {
    const bool v = (((reinterpret_cast<uintptr_t>(s) | reinterpret_cast<uintptr_t>(d) | bytes) & 15u) == 0);
    if (v) {
        const size_t nv = bytes / 16;
        for (size_t i = threadIdx.x; i < nv; i += kBflyThreads)
            st_v4(reinterpret_cast<uint4*>(d) + i, ld_cg_v4(reinterpret_cast<const uint4*>(s) + i));
    } else {
        for (size_t b = 2 * size_t(threadIdx.x); b < bytes; b += 2 * kBflyThreads)
            *reinterpret_cast<uint16_t*>(d + b) = ld_cg_u16(s + b);
    }
}

// Element range [lo, hi) of blocks [b0, b1) (blocks of `seg` elements, the last ones shorter).
__device__ __forceinline__ void block_range(const ButterflyArgs& a, int b0, int b1, size_t* lo, size_t* hi) {
    *lo = min(size_t(b0) * a.seg, a.n);
    *hi = min(size_t(b1) * a.seg, a.n);
}

template <int DT, int OP, bool SCALE, int KIND>
__global__ void __launch_bounds__(kBflyThreads, 2) k_butterfly(const __grid_constant__ ButterflyArgs a) {
    __shared__ uint32_t s_task;
    __shared__ int s_ok;
    const int p = a.p, L = a.log2p;
    const size_t d = size_t(Elem<DT>::kBytes);
    constexpr size_t kAcc = sizeof(typename Elem<DT>::A);
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
        const uint32_t rem = task - a.start[g];
        const int r = int(rem / a.ntile[g]);
        const uint32_t t = rem - uint32_t(r) * a.ntile[g];
        if (g > 0) {  // the previous step must be complete everywhere
            if (threadIdx.x == 0) {
                const unsigned long long want = a.start[g] - a.start[g - 1];
                s_ok = wait_counter(a.ctl, &a.st->step_ctr[g - 1], uint32_t(want), a.timeout_ns);
            }
            __syncthreads();
            if (!s_ok) break;
        }
        if constexpr (KIND == BFLY_RD) {
            const int dist = 1 << g, lo_r = min(r, r ^ dist), hi_r = max(r, r ^ dist);
            const size_t lo = min(size_t(t) * a.tile, a.n), hi = min(lo + a.tile, a.n);
            if (hi > lo) {
                auto vec_of = [&](int step, int rank) -> const char* {  // V_step[rank] at element lo
                    if (step == 0) return static_cast<const char*>(a.ptrs.send[rank]) + lo * d;
                    return a.stage + (size_t((step - 1) & 1) * p + rank) * a.stage_stride + lo * kAcc;
                };
                const bool last = (int(g) == L - 1);
                void* dst = last ? static_cast<void*>(static_cast<char*>(a.ptrs.recv[r]) + lo * d)
                                 : static_cast<void*>(a.stage + (size_t(g & 1) * p + r) * a.stage_stride + lo * kAcc);
                pair_reduce<DT, OP, SCALE>(vec_of(int(g), lo_r), g > 0, vec_of(int(g), hi_r), g > 0, dst, last,
                                           hi - lo, a.scale, a.vec != 0);
            }
        } else if (int(g) < L) {  // halving (reduce-scatter) step: distance p / 2^(g+1)
            const int dist = p >> (g + 1), partner = r ^ dist;
            const int lo_r = min(r, partner), hi_r = max(r, partner);
            const int group = (r / (2 * dist)) * (2 * dist);
            const int kb = (r & dist) ? group + dist : group;
            size_t klo, khi;
            block_range(a, kb, kb + dist, &klo, &khi);
            const size_t lo = min(klo + size_t(t) * a.tile, khi), hi = min(lo + a.tile, khi);
            if (hi > lo) {
                auto vec_of = [&](int rank) -> const char* {
                    if (g == 0) return static_cast<const char*>(a.ptrs.send[rank]) + lo * d;
                    return a.stage + size_t(rank) * a.stage_stride + lo * kAcc;
                };
                const bool last = (int(g) == L - 1);
                void* dst = last ? static_cast<void*>(static_cast<char*>(a.ptrs.recv[r]) + lo * d)
                                 : static_cast<void*>(a.stage + size_t(r) * a.stage_stride + lo * kAcc);
                pair_reduce<DT, OP, SCALE>(vec_of(lo_r), g > 0, vec_of(hi_r), g > 0, dst, last, hi - lo, a.scale,
                                           a.vec != 0);
            }
        } else {  // doubling (all-gather) step: distance 2^(g-L), copy the partner's block group
            const int dist = 1 << (int(g) - L), partner = r ^ dist;
            const int pg = (partner / dist) * dist;
            size_t klo, khi;
            block_range(a, pg, pg + dist, &klo, &khi);
            const size_t lo = min(klo + size_t(t) * a.tile, khi), hi = min(lo + a.tile, khi);
            if (hi > lo)
                bfly_copy(static_cast<const char*>(a.ptrs.recv[partner]) + lo * d,
                          static_cast<char*>(a.ptrs.recv[r]) + lo * d, (hi - lo) * d);
        }
        __syncthreads();
        if (threadIdx.x == 0 && r != a.skip_rank) {  // fault injection: one rank's tasks never count
            __threadfence();
            atomicAdd(&a.st->step_ctr[g], 1u);
        }
    }
    // Leave: the last CTA out resets the task counter and the step counters.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&a.st->done_ctr, 1u) == gridDim.x - 1) {
            a.st->task_ctr = 0;
            for (uint32_t g = 0; g < a.nsteps; ++g) a.st->step_ctr[g] = 0;
            a.st->done_ctr = 0;
            __threadfence();
        }
    }
}

template <int DT, int OP, bool SCALE>
static cudaError_t launch_kind(const ButterflyArgs& a, int ctas, cudaStream_t s) {
    if (a.kind == BFLY_RD) k_butterfly<DT, OP, SCALE, BFLY_RD><<<ctas, kBflyThreads, 0, s>>>(a);
    else k_butterfly<DT, OP, SCALE, BFLY_HD><<<ctas, kBflyThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <int DT>
static cudaError_t launch_dt(const ButterflyArgs& a, int op, int ctas, cudaStream_t s) {
    switch (op) {
        case COLL_SUM: return launch_kind<DT, COLL_SUM, false>(a, ctas, s);
        case COLL_MIN: return launch_kind<DT, COLL_MIN, false>(a, ctas, s);
        case COLL_MAX: return launch_kind<DT, COLL_MAX, false>(a, ctas, s);
        case COLL_AVG:
            if constexpr (DT == COLL_INT32) return cudaErrorInvalidValue;
            else return launch_kind<DT, COLL_SUM, true>(a, ctas, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_butterfly(const ButterflyArgs& a, int dtype, int op, int ctas, cudaStream_t s) {
    switch (dtype) {
        case COLL_INT32: return launch_dt<COLL_INT32>(a, op, ctas, s);
        case COLL_FP32: return launch_dt<COLL_FP32>(a, op, ctas, s);
        case COLL_BF16: return launch_dt<COLL_BF16>(a, op, ctas, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace simcomm
