// Copy engine: Broadcast, AllGather, All-to-All and All-to-Allv over TMA bulk copies.
//
// A collective is a list of segments (source range -> one or all ranks' destination ranges):
//   Broadcast  1 segment:   send[root]               -> recv[r]            for every r
//   AllGather  p segments:  send[q]                  -> recv[r] + q·m      for every r
//   All-to-All p² segments: send[i] + j·m            -> recv[j] + i·m
//   All-to-Allv p² segments: send[i] + sdispl[i][j]   -> recv[j] + rdispl[i][j], c[i][j] elements
// Segments are cut into tiles of at most kTile bytes whose interior lies on 16-byte boundaries.
// One warp per CTA runs a kStages-deep pipeline: one lane issues a cp.async.bulk load of a tile into
// shared memory (completing on an mbarrier), then one cp.async.bulk store per destination. A
// fan-out tile is thus read from HBM once and written p times. Bytes before the first and after
// the last 16-byte boundary, and segments whose source and destination disagree modulo 16, are
// copied by the warp with 2-byte loads and stores.
//
// Semantics ("集合通信：原语、算法、NCCL 实现与拓扑映射", llm-infra-atlas.github.io/hpc/04_collectives):
// §1.1 Broadcast, §1.2 AllGather (rank-ordered concatenation), §1.6 AllToAll (block transpose);
// All-to-Allv: "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All",
// section "Ragged All-to-All".
#include "a2av.cuh"
#include "common.cuh"
#include "tile_geom.h"

namespace simcomm {

constexpr int kCopyThreads = 32;
constexpr int kStages = 4;

static_assert(kStages <= 32, "stage phases live in one 32-bit mask");

struct SegDesc {
    const char* src;
    char* dst;        // single destination, or the base offset added to recv[r] for fan-out
    size_t dst_off;   // fan-out: offset in bytes into every recv[r]
    size_t len;       // bytes
    bool fanout;
};

template <int KIND>
__device__ __forceinline__ SegDesc segment(const CopyArgs& a, int s, const long long* sd, const long long* rd) {
    SegDesc d{};
    const size_t e = size_t(a.elem_bytes);
    if constexpr (KIND == COPY_BCAST) {
        d.src = static_cast<const char*>(a.ptrs.send[a.root]);
        d.fanout = true;
        d.dst_off = 0;
        d.len = a.blk_elems * e;
    } else if constexpr (KIND == COPY_ALLGATHER) {
        d.src = static_cast<const char*>(a.ptrs.send[s]);
        d.fanout = true;
        d.dst_off = size_t(s) * a.blk_elems * e;
        d.len = a.blk_elems * e;
    } else if constexpr (KIND == COPY_ALLTOALL) {
        const int i = s / a.p, j = s % a.p;
        d.src = static_cast<const char*>(a.ptrs.send[i]) + size_t(j) * a.blk_elems * e;
        d.dst = static_cast<char*>(a.ptrs.recv[j]) + size_t(i) * a.blk_elems * e;
        d.fanout = false;
        d.len = a.blk_elems * e;
    } else {
        const int i = s / a.p, j = s % a.p;
        d.src = static_cast<const char*>(a.ptrs.send[i]) + size_t(sd[s]) * e;
        d.dst = static_cast<char*>(a.ptrs.recv[j]) + size_t(rd[s]) * e;
        d.fanout = false;
        d.len = size_t(a.counts[s]) * e;
    }
    return d;
}

// A fan-out destination that is the source itself (in-place AllGather/Broadcast) is skipped.
__device__ __forceinline__ char* fan_dst(const CopyArgs& a, const SegDesc& d, int r) {
    return static_cast<char*>(a.ptrs.recv[r]) + d.dst_off;
}

__device__ __forceinline__ bool congruent(const CopyArgs& a, const SegDesc& d) {
    const uintptr_t delta = reinterpret_cast<uintptr_t>(d.src) & 15u;
    if (!d.fanout) return (reinterpret_cast<uintptr_t>(d.dst) & 15u) == delta;
    for (int r = 0; r < a.p; ++r)
        if ((reinterpret_cast<uintptr_t>(fan_dst(a, d, r)) & 15u) != delta) return false;
    return true;
}

// Warp copy of bytes [x, y) of a segment with 2-byte accesses (element sizes are 2 or 4 bytes,
// so every address and length here is even).
__device__ __forceinline__ void warp_copy_bytes(const CopyArgs& a, const SegDesc& d, size_t x, size_t y) {
    const int lane = threadIdx.x & 31;
    for (size_t b = x + 2 * size_t(lane); b < y; b += 64) {
        const uint16_t v = *reinterpret_cast<const uint16_t*>(d.src + b);
        if (d.fanout) {
            for (int r = 0; r < a.p; ++r) {
                char* dst = fan_dst(a, d, r);
                if (dst != d.src) *reinterpret_cast<uint16_t*>(dst + b) = v;
            }
        } else {
            *reinterpret_cast<uint16_t*>(d.dst + b) = v;
        }
    }
}

__device__ __forceinline__ int find_segment(const uint32_t* prefix, int nseg, uint32_t t) {
    int lo = 0, hi = nseg;  // invariant: prefix[lo] <= t < prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

template <int KIND>
__global__ void __launch_bounds__(kCopyThreads) k_copy(const __grid_constant__ CopyArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x;
    if (status_failed(a.ctl)) return;

    const int p = a.p;
    const int nseg = (KIND == COPY_BCAST) ? 1 : (KIND == COPY_ALLGATHER) ? p : p * p;
    unsigned char* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(kStages) * kTile);
    long long* sd = reinterpret_cast<long long*>(bars + kStages);
    long long* rd = sd + ((KIND == COPY_ALLTOALLV) ? p * p : 0);
    uint32_t* prefix = reinterpret_cast<uint32_t*>(rd + ((KIND == COPY_ALLTOALLV) ? p * p : 0));

    if constexpr (KIND == COPY_ALLTOALLV) {
        const A2avPlan plan = a2av_plan_warp(a.counts, p, a.send_cap, a.recv_cap, sd, rd, a.recv_counts_out, a.ctl);
        if (!plan.ok) return;
    }

    // tile counts per segment, then an inclusive scan into prefix[1..nseg]
    for (int s = lane; s < nseg; s += 32) {
        const SegDesc d = segment<KIND>(a, s, sd, rd);
        prefix[s + 1] = tile_count(reinterpret_cast<uintptr_t>(d.src), d.len, congruent(a, d));
    }
    __syncwarp();
    if (lane == 0) prefix[0] = 0;
    uint32_t carry = 0;
    for (int b = 0; b < nseg; b += 32) {
        const int s = b + lane;
        uint32_t v = (s < nseg) ? prefix[s + 1] : 0u;
#pragma unroll
        for (int dd = 1; dd < 32; dd <<= 1) {
            const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, v, dd);
            if (lane >= dd) v += o;
        }
        if (s < nseg) prefix[s + 1] = carry + v;
        carry += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
    __syncwarp();
    const uint32_t total = prefix[nseg];

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    __syncwarp();

    const uint32_t my_n = (total > blockIdx.x) ? (total - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    uint32_t phase = 0;  // bit s: parity of the next completion of stage s
    bool failed = false;

    auto issue = [&](uint32_t k) {
        const uint32_t t = blockIdx.x + k * gridDim.x;
        const int s = find_segment(prefix, nseg, t);
        const SegDesc d = segment<KIND>(a, s, sd, rd);
        const bool cong = congruent(a, d);
        const TileGeom g = tile_geom(reinterpret_cast<uintptr_t>(d.src), d.len, cong, t - prefix[s]);
        if (lane == 0 && g.bhi > g.blo) {
            const int st = int(k % kStages);
            mbar_arrive_expect_tx(&bars[st], uint32_t(g.bhi - g.blo));
            bulk_g2s(stages + size_t(st) * kTile, d.src + g.blo, uint32_t(g.bhi - g.blo), &bars[st]);
        }
    };

    auto consume = [&](uint32_t k) {
        const uint32_t t = blockIdx.x + k * gridDim.x;
        const int s = find_segment(prefix, nseg, t);
        const SegDesc d = segment<KIND>(a, s, sd, rd);
        const bool cong = congruent(a, d);
        const TileGeom g = tile_geom(reinterpret_cast<uintptr_t>(d.src), d.len, cong, t - prefix[s]);
        if (g.bhi > g.blo) {
            const int st = int(k % kStages);
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(a.ctl, &bars[st], (phase >> st) & 1u, a.timeout_ns);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            phase ^= (1u << st);
            if (!ok) { failed = true; return; }
            if (lane == 0) {
                fence_proxy_async_smem();
                const uint32_t bytes = uint32_t(g.bhi - g.blo);
                const unsigned char* src = stages + size_t(st) * kTile;
                if (d.fanout) {
                    for (int r = 0; r < p; ++r) {
                        char* dst = fan_dst(a, d, r);
                        if (dst != d.src) bulk_s2g(dst + g.blo, src, bytes);
                    }
                } else {
                    bulk_s2g(d.dst + g.blo, src, bytes);
                }
                bulk_commit();
            }
        }
        // head and tail bytes (or the whole tile when the segment is not 16-byte congruent)
        if (g.blo > g.lo) warp_copy_bytes(a, d, g.lo, g.blo);
        if (g.hi > g.bhi) warp_copy_bytes(a, d, g.bhi, g.hi);
    };

    const uint32_t pre = my_n < uint32_t(kStages - 1) ? my_n : uint32_t(kStages - 1);
    for (uint32_t k = 0; k < pre; ++k) issue(k);
    for (uint32_t k = 0; k < my_n && !failed; ++k) {
        const uint32_t kk = k + kStages - 1;
        if (kk < my_n) {
            // stage kk % kStages was last used by tile k-1, whose stores are the newest group
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            issue(kk);
        }
        consume(k);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
}

static size_t copy_smem_bytes(int kind, int p) {
    const int nseg = (kind == COPY_BCAST) ? 1 : (kind == COPY_ALLGATHER) ? p : p * p;
    size_t b = size_t(kStages) * kTile + size_t(kStages) * sizeof(uint64_t);
    if (kind == COPY_ALLTOALLV) b += 2 * size_t(p) * p * sizeof(long long);
    b += (size_t(nseg) + 1) * sizeof(uint32_t);
    return (b + 127) & ~size_t(127);
}

template <int KIND>
static cudaError_t launch_kind(const CopyArgs& a, int num_sms, cudaStream_t s) {
    const size_t smem = copy_smem_bytes(KIND, a.p);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_copy<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(copy_smem_bytes(KIND, kMaxRanks)));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    k_copy<KIND><<<num_sms, kCopyThreads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_copy(const CopyArgs& a, int num_sms, cudaStream_t s) {
    switch (a.kind) {
        case COPY_BCAST: return launch_kind<COPY_BCAST>(a, num_sms, s);
        case COPY_ALLGATHER: return launch_kind<COPY_ALLGATHER>(a, num_sms, s);
        case COPY_ALLTOALL: return launch_kind<COPY_ALLTOALL>(a, num_sms, s);
        case COPY_ALLTOALLV: return launch_kind<COPY_ALLTOALLV>(a, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace simcomm
