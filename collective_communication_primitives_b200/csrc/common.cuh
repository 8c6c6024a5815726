// Device-side building blocks shared by the simulated-communicator kernels (sm_100a).
//
// Memory access helpers are inline PTX: 16-byte streaming loads/stores, L2-coherent loads for
// data other CTAs produced in the same kernel, gpu-scope acquire/release flags, and the
// cp.async.bulk (TMA bulk copy) + mbarrier primitives of the copy engine. No multicast form of
// any bulk copy is used anywhere.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace simcomm {

// ---- element types -------------------------------------------------------------------------------

template <int DT> struct Elem;
template <> struct Elem<COLL_INT32> { using T = int32_t;  using A = int32_t; static constexpr int kBytes = 4; };
template <> struct Elem<COLL_FP32>  { using T = float;    using A = float;   static constexpr int kBytes = 4; };
template <> struct Elem<COLL_BF16>  { using T = uint16_t; using A = float;   static constexpr int kBytes = 2; };

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// fp32 -> bf16 round-to-nearest-even, via the CUDA intrinsic.
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

// The reduction operator: SUM (also used by AVG), MIN, MAX. MIN/MAX are written as a left fold
// that keeps the earlier operand on ties; int32 SUM wraps around.
template <int OP> __device__ __forceinline__ float op_f(float a, float b) {
    if (OP == COLL_MIN) return (b < a) ? b : a;
    if (OP == COLL_MAX) return (a < b) ? b : a;
    return a + b;
}
template <int OP> __device__ __forceinline__ int32_t op_i(int32_t a, int32_t b) {
    if (OP == COLL_MIN) return (b < a) ? b : a;
    if (OP == COLL_MAX) return (a < b) ? b : a;
    return int32_t(uint32_t(a) + uint32_t(b));
}

// ---- packs of W 32-bit words (W = 4: 16 bytes, W = 8: 32 bytes) --------------------------------
// A pack holds W fp32 / W int32 / 2W bf16 lanes, widened to the accumulator type.

template <int W> struct Words { uint32_t w[W]; };

template <int DT, int W> struct PackW;

template <int W> struct PackW<COLL_FP32, W> {
    static constexpr int L = W;
    using A = float;
    __device__ static void unpack(const Words<W>& v, float (&a)[L]) {
#pragma unroll
        for (int k = 0; k < W; ++k) a[k] = __uint_as_float(v.w[k]);
    }
    __device__ static Words<W> pack(const float (&a)[L]) {
        Words<W> v;
#pragma unroll
        for (int k = 0; k < W; ++k) v.w[k] = __float_as_uint(a[k]);
        return v;
    }
};

template <int W> struct PackW<COLL_INT32, W> {
    static constexpr int L = W;
    using A = int32_t;
    __device__ static void unpack(const Words<W>& v, int32_t (&a)[L]) {
#pragma unroll
        for (int k = 0; k < W; ++k) a[k] = int32_t(v.w[k]);
    }
    __device__ static Words<W> pack(const int32_t (&a)[L]) {
        Words<W> v;
#pragma unroll
        for (int k = 0; k < W; ++k) v.w[k] = uint32_t(a[k]);
        return v;
    }
};

template <int W> struct PackW<COLL_BF16, W> {
    static constexpr int L = 2 * W;
    using A = float;
    __device__ static void unpack(const Words<W>& v, float (&a)[L]) {
#pragma unroll
        for (int k = 0; k < W; ++k) {
            a[2 * k] = bf16_bits_to_float(v.w[k] & 0xFFFFu);
            a[2 * k + 1] = bf16_bits_to_float(v.w[k] >> 16);
        }
    }
    __device__ static Words<W> pack(const float (&a)[L]) {
        Words<W> v;
#pragma unroll
        for (int k = 0; k < W; ++k)
            v.w[k] = uint32_t(float_to_bf16_bits(a[2 * k])) | (uint32_t(float_to_bf16_bits(a[2 * k + 1])) << 16);
        return v;
    }
};

// 16-byte packs (the ring executor's unit).
template <int DT> struct Pack16 {
    using P = PackW<DT, 4>;
    static constexpr int L = P::L;
    using A = typename P::A;
    __device__ static void unpack(const uint4& v, A (&a)[L]) {
        Words<4> w{{v.x, v.y, v.z, v.w}};
        P::unpack(w, a);
    }
    __device__ static uint4 pack(const A (&a)[L]) {
        const Words<4> w = P::pack(a);
        return make_uint4(w.w[0], w.w[1], w.w[2], w.w[3]);
    }
};

template <int DT, int OP, typename A, int L>
__device__ __forceinline__ void fold_into(A (&acc)[L], const A (&x)[L]) {
#pragma unroll
    for (int l = 0; l < L; ++l) {
        if constexpr (DT == COLL_INT32) acc[l] = op_i<OP>(acc[l], x[l]);
        else acc[l] = op_f<OP>(acc[l], x[l]);
    }
}

// Element-wise access (plain loads: inputs are not written by the kernel that reads them).
template <int DT>
__device__ __forceinline__ typename Elem<DT>::A load_elem(const void* base, size_t e) {
    if constexpr (DT == COLL_BF16) return bf16_bits_to_float(static_cast<const uint16_t*>(base)[e]);
    else return static_cast<const typename Elem<DT>::T*>(base)[e];
}
template <int DT>
__device__ __forceinline__ void store_elem(void* base, size_t e, typename Elem<DT>::A v) {
    if constexpr (DT == COLL_BF16) static_cast<uint16_t*>(base)[e] = float_to_bf16_bits(v);
    else static_cast<typename Elem<DT>::T*>(base)[e] = v;
}

// ---- global memory access ------------------------------------------------------------------------

// Streaming 16-byte load of an input (not allocated in L1).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// 16-byte load through L2 only: for data that other CTAs wrote earlier in the same kernel.
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Streaming load / plain store of a pack of W words (W = 8 uses the 256-bit forms of sm_100).
template <int W> __device__ __forceinline__ Words<W> ld_stream_words(const void* p);
template <> __device__ __forceinline__ Words<4> ld_stream_words<4>(const void* p) {
    Words<4> v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]) : "l"(p));
    return v;
}
template <> __device__ __forceinline__ Words<8> ld_stream_words<8>(const void* p) {
    Words<8> v;
    asm volatile("ld.global.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
                   "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p));
    return v;
}
template <int W> __device__ __forceinline__ void st_words(void* p, const Words<W>& v);
template <> __device__ __forceinline__ void st_words<4>(void* p, const Words<4>& v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3])
                 : "memory");
}
template <> __device__ __forceinline__ void st_words<8>(void* p, const Words<8>& v) {
    asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
                    "r"(v.w[7])
                 : "memory");
}

__device__ __forceinline__ uint32_t ld_cg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint16_t ld_cg_u16(const void* p) {
    uint16_t v;
    asm volatile("ld.global.cg.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint8_t ld_cg_u8(const void* p) {
    uint32_t v;
    asm volatile("ld.global.cg.u8 %0, [%1];" : "=r"(v) : "l"(p));
    return uint8_t(v);
}

// ---- flags and status ------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_gpu_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
// Add v with release semantics and no return value (the thread does not wait for the L2 round trip).
__device__ __forceinline__ void red_release_add_gpu(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Record the first asynchronous error of the communicator: the device word decides the winner, the
// winner mirrors the code into the host-mapped word the host polls.
__device__ __forceinline__ void raise_status(const Ctl& ctl, uint32_t code) {
    if (atomicCAS(ctl.status, 0u, code) == 0u) {
        *ctl.host_status = code;
        __threadfence_system();
    }
}

__device__ __forceinline__ bool status_failed(const Ctl& ctl) {
    return *reinterpret_cast<volatile uint32_t*>(ctl.status) != 0u;
}

constexpr uint32_t kMaxSpin = 1u << 30;  // poll cap of every bounded wait (the timeout comes first)

// How a waiting thread polls (a build-time choice). Measured on B200: any __nanosleep in a wait
// loop (even 100 ns, or 1 us after a long wait) made a woken waiter notice its predecessor
// hundreds of microseconds late, turning every dependent ring step into a ~250 us stall; tight
// acquire polling (mode 0) was the fastest everywhere. Modes 2 and 3 remain for experiments.
//   0: acquire loads back to back (default);   1: relaxed loads, one acquire fence on success;
//   2: relaxed loads with a short sleep between polls;   3: acquire loads with a short sleep.
#ifndef SIMCOMM_WAIT_MODE
#define SIMCOMM_WAIT_MODE 0
#endif
#ifndef SIMCOMM_WAIT_SLEEP_NS
#define SIMCOMM_WAIT_SLEEP_NS 100
#endif

template <typename T> __device__ __forceinline__ T poll_load(const T* p);
template <> __device__ __forceinline__ unsigned long long poll_load(const unsigned long long* p) {
    return (SIMCOMM_WAIT_MODE == 0 || SIMCOMM_WAIT_MODE == 3) ? ld_acquire_gpu_u64(p) : ld_relaxed_gpu_u64(p);
}
template <> __device__ __forceinline__ uint32_t poll_load(const uint32_t* p) {
    return (SIMCOMM_WAIT_MODE == 0 || SIMCOMM_WAIT_MODE == 3) ? ld_acquire_gpu(p) : ld_relaxed_gpu(p);
}

// Whether the host asked for an abort. The host-mapped abort word is read by at most one waiter
// per kAbortPollNs on the whole GPU: the waiter that finds the shared clock stale and wins the CAS
// that advances it. (Measured on B200: when every one of ~300 waiting CTAs read host memory every
// 50 us, the CTAs doing the work slowed down 25-fold, e.g. a 63-hop Reduce chain of 1 MiB took
// 16.5 ms instead of 0.64 ms.)
constexpr uint64_t kAbortPollNs = 50000;
__device__ __forceinline__ bool abort_requested(const Ctl& ctl, uint64_t now) {
    const unsigned long long last = ld_relaxed_gpu_u64(ctl.abort_clock);
    if (int64_t(now - last) < int64_t(kAbortPollNs)) return false;
    if (atomicCAS(ctl.abort_clock, last, (unsigned long long)now) != last) return false;  // another waiter reads it
    return *ctl.abort_flag != 0u;
}

// Bounded wait until done(*p), called by one thread. Every 256 polls (policy above) the thread
// checks whether another CTA already failed, the global timer (timeout) and, rationed as above, the
// host-mapped abort word. Gives up (recording the reason) on failure, abort, timeout_ns of global
// time, or kMaxSpin polls. On success the caller's later loads see the producer's writes (acquire).
template <typename T, typename Done>
__device__ __forceinline__ bool bounded_wait(const Ctl& ctl, const T* p, Done done, uint64_t timeout_ns) {
    uint64_t t0 = 0;
    for (uint32_t it = 0; it < kMaxSpin; ++it) {
        if (done(poll_load(p))) {
            if (SIMCOMM_WAIT_MODE == 1 || SIMCOMM_WAIT_MODE == 2) fence_acq_rel_gpu();
            return true;
        }
        if (it == 0) {
            t0 = globaltimer_ns();
            continue;
        }
        if (SIMCOMM_WAIT_MODE >= 2) __nanosleep(SIMCOMM_WAIT_SLEEP_NS);
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

__device__ __forceinline__ bool wait_flag(const Ctl& ctl, const unsigned long long* flag, unsigned long long want,
                                          uint64_t timeout_ns) {
    return bounded_wait(ctl, flag, [want](unsigned long long v) { return v == want; }, timeout_ns);
}

// Bounded wait until a 32-bit counter reaches `want`.
__device__ __forceinline__ bool wait_counter(const Ctl& ctl, const uint32_t* ctr, uint32_t want, uint64_t timeout_ns) {
    return bounded_wait(ctl, ctr, [want](uint32_t v) { return v >= want; }, timeout_ns);
}

// Count one finished task of a chunk: the flag holds (epoch << 32) | tasks finished in this call;
// a flag left from an earlier call (older epoch) starts again at 1. The fence makes the CTA's
// writes (ordered before this call by a __syncthreads) visible before the count.
__device__ __forceinline__ void signal_chunk(const Ctl& ctl, unsigned long long* flag, uint32_t epoch) {
    __threadfence();
    const unsigned long long tag = (unsigned long long)epoch << 32;
    unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(flag);
    for (uint32_t it = 0; it < kMaxSpin; ++it) {
        const unsigned long long nv = ((v >> 32) == epoch) ? v + 1 : (tag | 1ull);
        const unsigned long long old = atomicCAS(flag, v, nv);
        if (old == v) return;
        v = old;
    }
    raise_status(ctl, COLL_ERR_INTERNAL);
}

// ---- dynamic task distribution ---------------------------------------------------------------------
// CTAs claim task numbers in increasing order from a counter in the communicator's scratch, so the
// tasks in flight at any moment are neighbours in the task order: for tasks laid out in address
// order, a narrow window of memory. (Measured on B200: a static grid-stride split of a stream over
// persistent CTAs reached 6.3 TB/s of stores where in-order distribution reached 7.4, and copies
// 6.4 against 6.9: with a static split the slowest CTA's share sets the end.) A CTA that finds the
// communicator failed claims nothing; every CTA that ran its task loop leaves through leave_tasks,
// and the last one to leave resets the counter for the next call.
__device__ __forceinline__ uint32_t claim_task(const Ctl& ctl, uint32_t* next, uint32_t total) {
    return status_failed(ctl) ? total : atomicAdd(next, 1u);
}

// Called by one thread per CTA after the CTA's last access to the counter.
__device__ __forceinline__ void leave_tasks(uint32_t* next, uint32_t* done) {
    __threadfence();
    if (atomicAdd(done, 1u) == gridDim.x * gridDim.y * gridDim.z - 1) {
        *next = 0;
        *done = 0;
        __threadfence();
    }
}

// ---- TMA bulk copies and mbarriers (shared::cta addresses, no multicast) -------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0u;
}
// Global -> shared bulk copy completing on an mbarrier. dst/src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// Shared -> global bulk copy tracked by bulk groups.
__device__ __forceinline__ void bulk_s2g(void* gdst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(gdst), "r"(smem_u32(smem_src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group has finished READING shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk group has completed (writes performed).
// Wait until at most the most recent bulk group is still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_but_last() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// L2 policy that evicts the touched lines first (streaming data read or written once).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar,
                                              uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        :: "r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(pol) : "memory");
}
__device__ __forceinline__ void bulk_s2g_hint(void* gdst, const void* smem_src, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 :: "l"(gdst), "r"(smem_u32(smem_src)), "r"(bytes), "l"(pol) : "memory");
}
// 16/32-byte streaming access with an L2 policy.
template <int W> __device__ __forceinline__ Words<W> ld_stream_words_hint(const void* p, uint64_t pol);
template <> __device__ __forceinline__ Words<4> ld_stream_words_hint<4>(const void* p, uint64_t pol) {
    Words<4> v;
    asm volatile("ld.global.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]) : "l"(p), "l"(pol));
    return v;
}
template <> __device__ __forceinline__ Words<8> ld_stream_words_hint<8>(const void* p, uint64_t pol) {
    Words<8> v;
    asm volatile("ld.global.L1::no_allocate.L2::cache_hint.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
                   "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p), "l"(pol));
    return v;
}
template <int W> __device__ __forceinline__ void st_words_hint(void* p, const Words<W>& v, uint64_t pol);
template <> __device__ __forceinline__ void st_words_hint<4>(void* p, const Words<4>& v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;"
                 :: "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "l"(pol) : "memory");
}
template <> __device__ __forceinline__ void st_words_hint<8>(void* p, const Words<8>& v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8}, %9;"
                 :: "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
                    "r"(v.w[6]), "r"(v.w[7]), "l"(pol)
                 : "memory");
}
// Streaming load/store of a pack, with (HINT) or without an evict-first L2 policy.
template <int W, bool HINT> __device__ __forceinline__ Words<W> ld_pack(const void* p, uint64_t pol) {
    if constexpr (HINT) return ld_stream_words_hint<W>(p, pol);
    else return ld_stream_words<W>(p);
}
template <int W, bool HINT> __device__ __forceinline__ void st_pack(void* p, const Words<W>& v, uint64_t pol) {
    if constexpr (HINT) st_words_hint<W>(p, v, pol);
    else st_words<W>(p, v);
}

// Bounded mbarrier wait; false (and a recorded error) if the phase never completes.
__device__ __forceinline__ bool mbar_wait_bounded(const Ctl& ctl, uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1; it < kMaxSpin; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0u && globaltimer_ns() - t0 > timeout_ns) break;
    }
    raise_status(ctl, COLL_ERR_INTERNAL);
    return false;
}

}  // namespace simcomm
