// HBM access-pattern probes: the bandwidth ceilings that the collectives' kernels are read against.
//
// Not a collective. Each probe streams one buffer (or two) through HBM with one access pattern of
// the library's kernels, so that a kernel's throughput can be compared with what that pattern can
// reach on the device: 32-byte loads alone (the fused reduction's input side), 32-byte stores alone,
// 32-byte load + store (a 1:1 copy), and bulk stores (cp.async.bulk shared -> global) of one
// shared-memory tile (the fan-out side of Broadcast and AllGather), and a bulk fan-out of every tile
// of one buffer to 8 copies (the whole Broadcast / AllGather pattern of 8 ranks).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace simcomm {

namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeUnroll = 4;
constexpr uint32_t kProbeTile = 16 * 1024;  // bytes of one bulk store
constexpr int kProbeBulkInFlight = 6;       // bulk store groups a CTA keeps in flight

template <int KIND>
__global__ void __launch_bounds__(kProbeThreads) k_probe_lsu(char* dst, const char* src, size_t nvec, uint32_t magic) {
    const size_t stride = size_t(gridDim.x) * kProbeThreads * kProbeUnroll;
    Words<8> pattern;
#pragma unroll
    for (int k = 0; k < 8; ++k) pattern.w[k] = 0x3C003C00u + uint32_t(k);
    uint32_t acc = 0;
    for (size_t v0 = size_t(blockIdx.x) * kProbeThreads * kProbeUnroll + threadIdx.x; v0 < nvec; v0 += stride) {
        Words<8> t[kProbeUnroll];
        if constexpr (KIND != PROBE_STORE) {
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u) {
                const size_t v = v0 + size_t(u) * kProbeThreads;
                if (v < nvec) t[u] = ld_stream_words<8>(src + v * 32);
            }
        }
        if constexpr (KIND == PROBE_LOAD) {
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u)
                if (v0 + size_t(u) * kProbeThreads < nvec) acc ^= t[u].w[0] ^ t[u].w[7];
        } else {
#pragma unroll
            for (int u = 0; u < kProbeUnroll; ++u) {
                const size_t v = v0 + size_t(u) * kProbeThreads;
                if (v < nvec) st_words<8>(dst + v * 32, KIND == PROBE_STORE ? pattern : t[u]);
            }
        }
    }
    // The loaded words feed a comparison with a value known only at run time, so the loads stay
    // live through the compiler's dead-code elimination; in the (practically never taken) equal case
    // the word goes to dst[0..3] when dst is given.
    if constexpr (KIND == PROBE_LOAD)
        if (acc == magic && dst) *reinterpret_cast<uint32_t*>(dst) = acc;
}

// One warp per CTA: a shared-memory tile stored over and over to consecutive 16 KiB pieces of dst.
__global__ void __launch_bounds__(32) k_probe_bulk_store(char* dst, size_t ntiles) {
    __shared__ __align__(128) unsigned char tile[kProbeTile];
    for (uint32_t b = threadIdx.x * 16; b < kProbeTile; b += 32 * 16)
        *reinterpret_cast<uint4*>(tile + b) = make_uint4(b, b + 1, b + 2, b + 3);
    fence_proxy_async_smem();
    __syncwarp();
    if (threadIdx.x != 0) return;
    uint32_t issued = 0;
    for (size_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        bulk_s2g(dst + t * kProbeTile, tile, kProbeTile);
        bulk_commit();
        if (++issued >= kProbeBulkInFlight)
            asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(kProbeBulkInFlight - 1) : "memory");
    }
    bulk_wait_all();
}

// Bulk fan-out 1:kProbeFan, the access pattern of a Broadcast or AllGather of kProbeFan ranks: every
// 32 KiB tile of src is loaded once into shared memory and stored to dst + f * bytes for each f (dst
// holds kProbeFan copies). One warp per CTA, kProbeFanStages tiles in flight, tiles claimed in order
// from a counter that the host clears before the launch.
constexpr int kProbeFan = 8;
constexpr int kProbeFanStages = 4;
constexpr uint32_t kProbeFanTile = 32 * 1024;
constexpr uint64_t kProbeWaitNs = 1000000000ull;  // 1 s
__device__ uint32_t g_probe_ctr;

__global__ void __launch_bounds__(32) k_probe_fanout(char* dst, const char* src, size_t bytes, uint32_t ntiles) {
    extern __shared__ __align__(128) unsigned char stages[];
    __shared__ uint64_t bars[kProbeFanStages];
    __shared__ uint32_t tiles[kProbeFanStages];
    if (threadIdx.x != 0) return;
    for (int st = 0; st < kProbeFanStages; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
    uint32_t phase = 0, head = 0, tail = 0;
    bool more = true;
    auto issue = [&]() {
        const uint32_t t = atomicAdd(&g_probe_ctr, 1u);
        if (t >= ntiles) {
            more = false;
            return;
        }
        const int st = int(head % kProbeFanStages);
        tiles[st] = t;
        mbar_arrive_expect_tx(&bars[st], kProbeFanTile);
        bulk_g2s(stages + size_t(st) * kProbeFanTile, src + size_t(t) * kProbeFanTile, kProbeFanTile, &bars[st]);
        ++head;
    };
    while (more && head < kProbeFanStages - 1) issue();
    while (tail < head) {
        const int st = int(tail % kProbeFanStages);
        // a load that has not landed after kProbeWaitNs of global time ends the probe (the probe has
        // no error channel; its caller sees the time, not the data)
        bool ok = mbar_try_wait(&bars[st], (phase >> st) & 1u);
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 1; !ok && it < kMaxSpin; ++it) {
            ok = mbar_try_wait(&bars[st], (phase >> st) & 1u);
            if (!ok && (it & 255u) == 0u && globaltimer_ns() - t0 > kProbeWaitNs) break;
        }
        if (!ok) break;
        phase ^= 1u << st;
        for (int f = 0; f < kProbeFan; ++f)
            bulk_s2g(dst + size_t(f) * bytes + size_t(tiles[st]) * kProbeFanTile, stages + size_t(st) * kProbeFanTile,
                     kProbeFanTile);
        bulk_commit();
        ++tail;
        if (more) {
            bulk_wait_read_all();
            issue();
        }
    }
    bulk_wait_all();
}

}  // namespace

cudaError_t launch_probe(int kind, void* dst, const void* src, size_t bytes, int ctas_per_sm, int num_sms,
                         cudaStream_t s) {
    if (kind == PROBE_BULK_FANOUT) {
        const uint32_t ntiles = uint32_t(bytes / kProbeFanTile);
        void* ctr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ctr, g_probe_ctr);
        if (e == cudaSuccess) e = cudaMemsetAsync(ctr, 0, sizeof(uint32_t), s);
        const size_t smem = size_t(kProbeFanStages) * kProbeFanTile;
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_probe_fanout, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        const size_t grid = std::min<size_t>(size_t(num_sms) * std::max(ctas_per_sm, 1), std::max<uint32_t>(ntiles, 1u));
        k_probe_fanout<<<unsigned(grid), 32, smem, s>>>(static_cast<char*>(dst), static_cast<const char*>(src), bytes,
                                                      ntiles);
        return cudaGetLastError();
    }
    if (kind == PROBE_BULK_STORE) {
        const size_t ntiles = bytes / kProbeTile;
        const size_t want = std::max<size_t>(ntiles, 1);  // one pass: a CTA per tile
        const size_t grid = ctas_per_sm > 0 ? std::min<size_t>(size_t(num_sms) * ctas_per_sm, want) : want;
        k_probe_bulk_store<<<unsigned(grid), 32, 0, s>>>(static_cast<char*>(dst), ntiles);
        return cudaGetLastError();
    }
    const size_t nvec = bytes / 32;
    const size_t per_cta = size_t(kProbeThreads) * kProbeUnroll;
    const size_t want = std::max<size_t>((nvec + per_cta - 1) / per_cta, 1);  // one pass: a CTA per iteration
    const size_t grid = ctas_per_sm > 0 ? std::min<size_t>(size_t(num_sms) * ctas_per_sm, want) : want;
    char* d = static_cast<char*>(dst);
    const char* x = static_cast<const char*>(src);
    switch (kind) {
        case PROBE_LOAD: k_probe_lsu<PROBE_LOAD><<<unsigned(grid), kProbeThreads, 0, s>>>(d, x, nvec, 0x9E3779B9u); break;
        case PROBE_STORE: k_probe_lsu<PROBE_STORE><<<unsigned(grid), kProbeThreads, 0, s>>>(d, x, nvec, 0x9E3779B9u); break;
        case PROBE_COPY: k_probe_lsu<PROBE_COPY><<<unsigned(grid), kProbeThreads, 0, s>>>(d, x, nvec, 0x9E3779B9u); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace simcomm
