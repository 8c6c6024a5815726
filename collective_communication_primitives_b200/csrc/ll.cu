// Low-latency (LL) ring and recursive-doubling AllReduce: the flag travels inside the data.
//
// "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives), §3.4
// protocols: the Simple protocol moves data and then raises a separate flag behind a memory fence;
// LL puts a flag beside every 4 bytes of data in one 8-byte store, so the receiver polls the data
// itself and the sender needs no fence, at half the bandwidth; it serves small messages. (LL128 puts
// 8 bytes of flag in every 128-byte line; it is not built here.)
// Schedule and arithmetic are those of the ring AllReduce (§2.2, our reading of the garbled trace):
// reduce-scatter step s = 1..p-1, rank r computes segment (r-1-s) mod p as received ⊕ own, partials
// in fp32 for fp32/bf16 data, the owner scales for AVG and rounds once; all-gather step s = 1..p-1,
// rank r receives segment (r-s) mod p from rank r-1. Its result therefore equals the ring path's bit
// for bit.
//
// Execution: one cooperative launch (every CTA resident at once, so waiting on another CTA always
// ends). CTAs [r*G, (r+1)*G) play rank r; thread t of rank r owns the same element positions of
// every segment, and at every step needs only what thread t of rank r-1 produced the step before,
// so threads never synchronise with each other. A value crosses a hop as one 64-bit store
// (tag << 32 | value bits) into the receiver's slot for that step; the receiver polls those 64 bits
// until the tag is this call's tag for that step (bounded, like every wait). The first hop reads the
// predecessor's input in place.
#include "common.cuh"

namespace simcomm {

constexpr int kLLThreads = 256;

__device__ __forceinline__ void st_relaxed_gpu_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}

// Wait until the slot holds this step's tag; returns its 32 data bits through *val.
__device__ __forceinline__ bool ll_wait(const Ctl& ctl, const unsigned long long* w, uint32_t tag, uint64_t timeout_ns,
                                        uint32_t* val) {
    uint64_t t0 = 0;
    for (uint32_t it = 0; it < kMaxSpin; ++it) {
        const unsigned long long v = ld_relaxed_gpu_u64(w);
        if (uint32_t(v >> 32) == tag) {
            *val = uint32_t(v);
            return true;
        }
        if (it == 0) {
            t0 = globaltimer_ns();
            continue;
        }
        if ((it & 255u) == 0u) {
            if (status_failed(ctl)) return false;
            const uint64_t now = globaltimer_ns();
            if (now - t0 > timeout_ns) { raise_status(ctl, COLL_ERR_TIMEOUT); return false; }
            if (abort_requested(ctl, now)) { raise_status(ctl, COLL_ERR_ABORTED); return false; }
        }
    }
    raise_status(ctl, COLL_ERR_TIMEOUT);
    return false;
}

template <int DT>
__device__ __forceinline__ uint32_t acc_bits(typename Elem<DT>::A v) {
    if constexpr (DT == COLL_INT32) return uint32_t(v);
    else return __float_as_uint(v);
}
template <int DT>
__device__ __forceinline__ typename Elem<DT>::A acc_of(uint32_t b) {
    if constexpr (DT == COLL_INT32) return int32_t(b);
    else return __uint_as_float(b);
}
// The element's output bits (the rounded value) and back.
template <int DT>
__device__ __forceinline__ uint32_t out_bits(typename Elem<DT>::A v) {
    if constexpr (DT == COLL_BF16) return uint32_t(float_to_bf16_bits(v));
    else if constexpr (DT == COLL_FP32) return __float_as_uint(v);
    else return uint32_t(v);
}
template <int DT>
__device__ __forceinline__ void store_bits(void* base, size_t e, uint32_t b) {
    if constexpr (DT == COLL_BF16) static_cast<uint16_t*>(base)[e] = uint16_t(b);
    else static_cast<uint32_t*>(base)[e] = b;
}

// The element's bits as stored (bf16: 16 bits, fp32/int32: 32 bits).
template <int DT>
__device__ __forceinline__ uint32_t raw_bits(const void* base, size_t e) {
    if constexpr (DT == COLL_BF16) return static_cast<const uint16_t*>(base)[e];
    else return static_cast<const uint32_t*>(base)[e];
}

// MODE LL_RING (AllReduce): the reduce-scatter steps then the all-gather steps; slots: reduce-scatter
// step s (2..p-1) in slot s-2, all-gather step s (1..p-1) in slot p-2+s-1. MODE LL_RING_RS
// (ReduceScatter): the reduce-scatter steps only, the owner's segment written to its output at
// offset 0. MODE LL_RING_AG (AllGather): the all-gather steps only, the input being the rank's own
// segment: step 1 reads the predecessor's input in place, steps s >= 2 go through slot s-2.
template <int DT, int OP, bool SCALE, int MODE>
__global__ void __launch_bounds__(kLLThreads) k_ring_ll(const __grid_constant__ LLArgs a) {
    using A = typename Elem<DT>::A;
    const int p = a.p;
    const int r = int(blockIdx.x) / a.G;
    const int pred = (r + p - 1) % p;
    const size_t i0 = size_t(int(blockIdx.x) % a.G) * kLLThreads + threadIdx.x;
    const size_t stride = size_t(a.G) * kLLThreads;
    unsigned long long* mine = a.ll + size_t(r) * a.nslots * a.seg;
    unsigned long long* next = a.ll + size_t((r + 1) % p) * a.nslots * a.seg;
    if (status_failed(a.ctl)) return;
    auto seg_of = [&](int s) { return ((r - s) % p + p) % p; };  // rank r's segment at all-gather step s
    auto word = [&](uint32_t q, uint32_t bits) { return ((unsigned long long)(a.tag + q) << 32) | bits; };
    if constexpr (MODE != LL_RING_AG) {
        for (int s = 1; s <= p - 1; ++s) {  // reduce-scatter: segment (r-1-s) mod p = received ⊕ own
            const int k = ((r - 1 - s) % p + p) % p;
            for (size_t i = i0; i < a.seg; i += stride) {
                const size_t e = size_t(k) * a.seg + i;
                if (e >= a.n) break;
                A w;
                if (s == 1) {
                    w = load_elem<DT>(a.ptrs.send[pred], e);
                } else {
                    uint32_t b;
                    if (!ll_wait(a.ctl, mine + size_t(s - 2) * a.seg + i, a.tag + uint32_t(s - 2), a.timeout_ns, &b))
                        return;
                    w = acc_of<DT>(b);
                }
                const A o = load_elem<DT>(a.ptrs.send[r], e);
                if constexpr (DT == COLL_INT32) w = op_i<OP>(w, o);
                else w = op_f<OP>(w, o);
                if (s < p - 1) {
                    const uint32_t q = uint32_t(s - 1);  // the successor's slot for step s+1
                    if (r != a.skip_rank) st_relaxed_gpu_u64(next + size_t(q) * a.seg + i, word(q, acc_bits<DT>(w)));
                } else {
                    if constexpr (SCALE) w = w * a.scale;
                    const uint32_t ob = out_bits<DT>(w);
                    if constexpr (MODE == LL_RING_RS) {
                        store_bits<DT>(a.ptrs.recv[r], i, ob);  // k == r: the owner's segment
                    } else {
                        store_bits<DT>(a.ptrs.recv[r], e, ob);
                        const uint32_t q = uint32_t(p - 2);  // the successor's slot for all-gather step 1
                        if (r != a.skip_rank) st_relaxed_gpu_u64(next + size_t(q) * a.seg + i, word(q, ob));
                    }
                }
            }
        }
    }
    if constexpr (MODE != LL_RING_RS) {
        if constexpr (MODE == LL_RING_AG) {  // the own segment into the own output
            for (size_t i = i0; i < a.seg; i += stride) {
                const size_t e = size_t(r) * a.seg + i;
                if (e >= a.n) break;
                store_bits<DT>(a.ptrs.recv[r], e, raw_bits<DT>(a.ptrs.send[r], i));
            }
        }
        for (int s = 1; s <= p - 1; ++s) {  // all-gather: segment (r-s) mod p from rank r-1
            const int k = seg_of(s);
            // this step's slot (unused when AllGather's first step reads in place) and the next one's
            const int q_in = (MODE == LL_RING_AG) ? s - 2 : p - 2 + s - 1;
            const uint32_t q_out = uint32_t(q_in + 1);
            for (size_t i = i0; i < a.seg; i += stride) {
                const size_t e = size_t(k) * a.seg + i;
                if (e >= a.n) break;
                uint32_t b;
                if (MODE == LL_RING_AG && s == 1) {
                    b = raw_bits<DT>(a.ptrs.send[pred], i);  // the predecessor's own segment, in place
                } else if (!ll_wait(a.ctl, mine + size_t(q_in) * a.seg + i, a.tag + uint32_t(q_in), a.timeout_ns, &b)) {
                    return;
                }
                store_bits<DT>(a.ptrs.recv[r], e, b);
                if (s < p - 1 && r != a.skip_rank) st_relaxed_gpu_u64(next + size_t(q_out) * a.seg + i, word(q_out, b));
            }
        }
    }
}

// Recursive doubling on the LL protocol ("集合通信：原语、算法、NCCL 实现与拓扑映射" §2.3 schedule,
// §3.4 protocol): log2 p steps; at step k every rank sends its whole partial vector to the rank at
// distance 2^k and combines the two, the lower rank's value first (the same arithmetic as the
// butterfly executor's recursive doubling, so the same bits). Thread t of rank r keeps EPT of its
// rank's elements (t, t + S, ..., S = threads per rank) in registers across the steps; at each step
// it first stores all of them into the partner's slot for that step, then polls its own slot for the
// partner's values, so two partners never wait on each other in a cycle.
template <int DT, int OP, bool SCALE, int EPT>
__global__ void __launch_bounds__(kLLThreads) k_rd_ll(const __grid_constant__ LLArgs a) {
    using A = typename Elem<DT>::A;
    const int p = a.p;
    const int r = int(blockIdx.x) / a.G;
    const size_t S = size_t(a.G) * kLLThreads;
    const size_t t0 = size_t(int(blockIdx.x) % a.G) * kLLThreads + threadIdx.x;
    if (status_failed(a.ctl)) return;
    A v[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        const size_t e = t0 + size_t(j) * S;
        v[j] = (e < a.n) ? load_elem<DT>(a.ptrs.send[r], e) : A(0);
    }
    for (int k = 0; (1 << k) < p; ++k) {
        const int q = r ^ (1 << k);
        const uint32_t tag = a.tag + uint32_t(k);
        unsigned long long* theirs = a.ll + (size_t(q) * a.nslots + k) * a.n;
        const unsigned long long* mine = a.ll + (size_t(r) * a.nslots + k) * a.n;
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const size_t e = t0 + size_t(j) * S;
            if (e < a.n && r != a.skip_rank) st_relaxed_gpu_u64(theirs + e, ((unsigned long long)tag << 32) | acc_bits<DT>(v[j]));
        }
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const size_t e = t0 + size_t(j) * S;
            if (e >= a.n) continue;
            uint32_t b;
            if (!ll_wait(a.ctl, mine + e, tag, a.timeout_ns, &b)) return;
            const A w = acc_of<DT>(b);
            const A lo = (r < q) ? v[j] : w, hi = (r < q) ? w : v[j];
            if constexpr (DT == COLL_INT32) v[j] = op_i<OP>(lo, hi);
            else v[j] = op_f<OP>(lo, hi);
        }
    }
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        const size_t e = t0 + size_t(j) * S;
        if (e >= a.n) continue;
        A x = v[j];
        if constexpr (SCALE) x = x * a.scale;
        store_bits<DT>(a.ptrs.recv[r], e, out_bits<DT>(x));
    }
}

// The binary tree on the LL protocol ("Collective Communication：…" "Tree AllReduce 为什么更适合延迟
// 敏感区间": reduce up a tree, broadcast down; the same heap tree and fold as the tree executor's
// single tree, so the same bits): position m holds rank m, children 2m+1 and 2m+2. Rank r's slots:
// 0 and 1 receive its left and right child's partial, 2 receives its parent's result. Thread t of
// every rank owns the same elements; per element a position waits for its children's words (a leaf
// for none), folds (own ⊕ left) ⊕ right, and sends the partial to its parent (the root instead
// scales, rounds and writes its output); then it waits for its parent's result (the root for none),
// writes it and forwards it to its children. Every wait is on a deeper position (reduce) or a
// shallower one (broadcast), so no two threads wait on each other in a cycle. The double tree
// ([Atlas] §2.4) runs the second half of the elements over the mirror tree in CTAs of their own.
template <int DT, int OP, bool SCALE>
__global__ void __launch_bounds__(kLLThreads) k_tree_ll(const __grid_constant__ LLArgs a) {
    using A = typename Elem<DT>::A;
    const int p = a.p;
    const int r = int(blockIdx.x) / a.G;
    const int g = int(blockIdx.x) % a.G;
    // The double tree: CTAs [0, GA) of a rank carry tree A's elements [0, seg) (rank m at heap
    // position m), the others tree B's [seg, n) (the mirror: rank m at position p - 1 - m). The single
    // tree has GA = G and seg = n. A CTA serves one tree, so every lane of a warp holds the same
    // position: lanes never wait on each other's sends through a warp's reconvergence.
    const bool tb = g >= a.GA;
    const size_t lo = tb ? a.seg : 0, hi = tb ? a.n : a.seg;
    const size_t i0 = lo + size_t(tb ? g - a.GA : g) * kLLThreads + threadIdx.x;
    const size_t stride = size_t(tb ? a.G - a.GA : a.GA) * kLLThreads;
    if (status_failed(a.ctl)) return;
    const int pos = tb ? p - 1 - r : r;
    auto rank_at = [&](int q) { return tb ? p - 1 - q : q; };
    const unsigned long long* mine = a.ll + size_t(r) * a.nslots * a.n;
    auto slot_of = [&](int rank, int q) { return a.ll + (size_t(rank) * a.nslots + q) * a.n; };
    const bool silent = (r == a.skip_rank);
    const int ppos = (pos - 1) / 2;
    const int side = (pos == 2 * ppos + 1) ? 0 : 1;  // which child of its parent this position is
    // reduce up
    for (size_t e = i0; e < hi; e += stride) {
        A x = load_elem<DT>(a.ptrs.send[r], e);
        for (int c = 0; c < 2; ++c) {
            if (2 * pos + 1 + c >= p) break;
            uint32_t b;
            if (!ll_wait(a.ctl, mine + size_t(c) * a.n + e, a.tag + uint32_t(c), a.timeout_ns, &b)) return;
            if constexpr (DT == COLL_INT32) x = op_i<OP>(x, acc_of<DT>(b));
            else x = op_f<OP>(x, acc_of<DT>(b));
        }
        if (pos == 0) {
            if constexpr (SCALE) x = x * a.scale;
            const uint32_t ob = out_bits<DT>(x);
            store_bits<DT>(a.ptrs.recv[r], e, ob);
            for (int c = 0; c < 2; ++c) {  // the result starts down the tree
                if (1 + c < p && !silent)
                    st_relaxed_gpu_u64(slot_of(rank_at(1 + c), 2) + e, ((unsigned long long)(a.tag + 2u) << 32) | ob);
            }
        } else if (!silent) {
            st_relaxed_gpu_u64(slot_of(rank_at(ppos), side) + e,
                               ((unsigned long long)(a.tag + uint32_t(side)) << 32) | acc_bits<DT>(x));
        }
    }
    if (pos == 0) return;
    // broadcast down
    for (size_t e = i0; e < hi; e += stride) {
        uint32_t b;
        if (!ll_wait(a.ctl, mine + size_t(2) * a.n + e, a.tag + 2u, a.timeout_ns, &b)) return;
        store_bits<DT>(a.ptrs.recv[r], e, b);
        for (int c = 0; c < 2; ++c) {
            const int kp = 2 * pos + 1 + c;
            if (kp < p && !silent)
                st_relaxed_gpu_u64(slot_of(rank_at(kp), 2) + e, ((unsigned long long)(a.tag + 2u) << 32) | b);
        }
    }
}

template <int DT, int OP, bool SCALE>
static cudaError_t launch_ll_typed(const LLArgs& a, cudaStream_t s) {
    void* args[] = {const_cast<LLArgs*>(&a)};
    const void* f = reinterpret_cast<const void*>(&k_ring_ll<DT, OP, SCALE, LL_RING>);
    if (a.kind == LL_RING_RS) f = reinterpret_cast<const void*>(&k_ring_ll<DT, OP, SCALE, LL_RING_RS>);
    if (a.kind == LL_RING_AG) f = reinterpret_cast<const void*>(&k_ring_ll<DT, OP, SCALE, LL_RING_AG>);
    if (a.kind == LL_TREE) f = reinterpret_cast<const void*>(&k_tree_ll<DT, OP, SCALE>);
    if (a.kind == LL_RD) {
        switch (a.ept) {
            case 1: f = reinterpret_cast<const void*>(&k_rd_ll<DT, OP, SCALE, 1>); break;
            case 2: f = reinterpret_cast<const void*>(&k_rd_ll<DT, OP, SCALE, 2>); break;
            case 4: f = reinterpret_cast<const void*>(&k_rd_ll<DT, OP, SCALE, 4>); break;
            case 8: f = reinterpret_cast<const void*>(&k_rd_ll<DT, OP, SCALE, 8>); break;
            default: return cudaErrorInvalidValue;
        }
    }
    return cudaLaunchCooperativeKernel(f, dim3(unsigned(a.p * a.G)), dim3(kLLThreads), args, 0, s);
}

template <int DT>
static cudaError_t launch_ll_dt(const LLArgs& a, int op, cudaStream_t s) {
    switch (op) {
        case COLL_SUM: return launch_ll_typed<DT, COLL_SUM, false>(a, s);
        case COLL_MIN: return launch_ll_typed<DT, COLL_MIN, false>(a, s);
        case COLL_MAX: return launch_ll_typed<DT, COLL_MAX, false>(a, s);
        case COLL_AVG:
            if constexpr (DT == COLL_INT32) return cudaErrorInvalidValue;
            else return launch_ll_typed<DT, COLL_SUM, true>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_ring_ll(const LLArgs& a, int dtype, int op, cudaStream_t s) {
    switch (dtype) {
        case COLL_INT32: return launch_ll_dt<COLL_INT32>(a, op, s);
        case COLL_FP32: return launch_ll_dt<COLL_FP32>(a, op, s);
        case COLL_BF16: return launch_ll_dt<COLL_BF16>(a, op, s);
        default: return cudaErrorInvalidValue;
    }
}

// CTAs of the LL kernels that fit on the device at once (the cooperative-launch limit; the kernel
// with the most registers sets it).
int ring_ll_max_ctas(int num_sms) {
    int a = 0, b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&a, k_ring_ll<COLL_BF16, COLL_SUM, true, LL_RING>, kLLThreads, 0) !=
            cudaSuccess || a < 1)
        a = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_rd_ll<COLL_FP32, COLL_SUM, true, 8>, kLLThreads, 0) !=
            cudaSuccess || b < 1)
        b = 1;
    return num_sms * (a < b ? a : b);
}

}  // namespace simcomm
