// Copy engine: Broadcast, AllGather, All-to-All, All-to-Allv, Scatter and Gather over TMA bulk copies.
//
// A collective is a list of segments (source range -> one or all ranks' destination ranges):
//   Broadcast  1 segment:   send[root]               -> recv[r]            for every r
//   AllGather  p segments:  send[q]                  -> recv[r] + q·m      for every r
//   All-to-All p² segments: send[i] + j·m            -> recv[j] + i·m
//   All-to-Allv p² segments: send[i] + sdispl[i][j]   -> recv[j] + rdispl[i][j], c[i][j] elements
//   Scatter    p segments:  send[root] + r·m         -> recv[r]
//   Gather     p segments:  send[r]                  -> recv[root] + r·m
// Segments are cut into tiles of at most kTile bytes whose interior lies on 16-byte boundaries.
// One warp per CTA runs a kStages-deep pipeline: one lane issues a cp.async.bulk load of a tile into
// shared memory (completing on an mbarrier), then one cp.async.bulk store per destination. A
// fan-out tile is thus read from HBM once and written p times. Bytes before the first and after
// the last 16-byte boundary, and segments whose source and destination disagree modulo 16, are
// copied by the warp with 2-byte loads and stores. On aligned buffers Broadcast, AllGather and the
// equal All-to-All take a lean form of the same pipeline (k_fanout: whole 32 KiB tiles, one lane,
// nothing else on its path), and the equal All-to-All can also run as one pass of 32-byte loads
// and stores (k_a2a_pass); All-to-All(v) also has a 16-byte load/store path (k_copy_lsu).
//
// Semantics ("集合通信：原语、算法、NCCL 实现与拓扑映射", llm-infra-atlas.github.io/hpc/04_collectives):
// §1.1 Broadcast, §1.2 AllGather (rank-ordered concatenation), §1.6 AllToAll (block transpose);
// All-to-Allv: "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All",
// section "Ragged All-to-All".
#include "a2av.cuh"
#include "common.cuh"
#include "tile_geom.h"

#include <algorithm>

namespace simcomm {

constexpr int kCopyThreads = 32;

// Pipeline shapes (stages x tile bytes, CTAs per SM), selected with the "copy_variant" option.
struct CopyShape { int stages; uint32_t tile; int ctas_per_sm; };
constexpr CopyShape kCopyShapes[] = {
    {4, 32768, 1}, {6, 32768, 1}, {3, 65536, 1}, {2, 65536, 1},
    {4, 16384, 2}, {6, 16384, 2}, {2, 32768, 3}, {8, 16384, 1},
};
constexpr int kNumCopyShapes = int(sizeof(kCopyShapes) / sizeof(kCopyShapes[0]));

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
    } else if constexpr (KIND == COPY_SCATTER) {
        d.src = static_cast<const char*>(a.ptrs.send[a.root]) + size_t(s) * a.blk_elems * e;
        d.dst = static_cast<char*>(a.ptrs.recv[s]);
        d.fanout = false;
        d.len = (d.src == d.dst) ? 0 : a.blk_elems * e;  // in place: the root's block stays
    } else if constexpr (KIND == COPY_GATHER) {
        d.src = static_cast<const char*>(a.ptrs.send[s]);
        d.dst = static_cast<char*>(a.ptrs.recv[a.root]) + size_t(s) * a.blk_elems * e;
        d.fanout = false;
        d.len = (d.src == d.dst) ? 0 : a.blk_elems * e;
    } else {
        // a rank view's All-to-Allv has the p blocks bound for its own rank only: segment s is the
        // block from source s
        const int ij = a.only_dst_plus1 ? s * a.p + (a.only_dst_plus1 - 1) : s;
        const int i = ij / a.p, j = ij % a.p;
        d.src = static_cast<const char*>(a.ptrs.send[i]) + size_t(sd[ij]) * e;
        d.dst = static_cast<char*>(a.ptrs.recv[j]) + size_t(rd[ij]) * e;
        d.fanout = false;
        d.len = size_t(a.counts[ij]) * e;
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

// ---- interleaved task order over blocks of unequal size --------------------------------------------
// Level k holds tile k of every block that has more than k tiles; the interleaved order runs the
// levels one after another, blocks in index order within a level. With blocks of equal size that is
// t -> (block t % nseg, tile t / nseg); with unequal ones (skewed All-to-Allv counts) a table of the
// first task of every level maps a task to its level, and a ballot over the blocks finds its block,
// so no slot is empty and every CTA gets an equal share of real tasks.
constexpr int kMaxLevels = 8192;

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += o;
    }
    return v;
}

// lvl[k], k = 0..tmax: tasks on the levels below k. prefix[s+1] - prefix[s] = tiles of block s, at most
// tmax. One full warp.
__device__ void build_levels(const uint32_t* prefix, int nseg, uint32_t tmax, uint32_t* lvl, int lane) {
    for (uint32_t v = lane; v <= tmax; v += 32) lvl[v] = 0;
    __syncwarp();
    for (int s = lane; s < nseg; s += 32) atomicAdd(&lvl[prefix[s + 1] - prefix[s]], 1u);  // blocks per tile count
    __syncwarp();
    uint32_t carry_c = 0, carry_l = 0;
    for (uint32_t b = 0; b <= tmax; b += 32) {
        const uint32_t v = b + uint32_t(lane);
        const uint32_t h = v <= tmax ? lvl[v] : 0u;
        const uint32_t hs = warp_incl_scan(h, lane);
        const uint32_t act = v <= tmax ? uint32_t(nseg) - (carry_c + hs) : 0u;  // blocks with more than v tiles
        const uint32_t ls = warp_incl_scan(act, lane);
        __syncwarp();
        if (v <= tmax) lvl[v] = carry_l + ls - act;
        carry_c += __shfl_sync(0xFFFFFFFFu, hs, 31);
        carry_l += __shfl_sync(0xFFFFFFFFu, ls, 31);
    }
    __syncwarp();
}

// The j-th block (in index order) of those with more than lv tiles. One full warp.
__device__ __forceinline__ int level_pick(const uint32_t* prefix, int nseg, uint32_t lv, uint32_t j, int lane) {
    for (int b = 0; b < nseg; b += 32) {
        const int s = b + lane;
        const bool act = s < nseg && prefix[s + 1] - prefix[s] > lv;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, act);
        const uint32_t c = uint32_t(__popc(m));
        if (j < c) {
            const bool me = act && uint32_t(__popc(m & ((1u << lane) - 1u))) == j;
            return b + __ffs(__ballot_sync(0xFFFFFFFFu, me)) - 1;
        }
        j -= c;
    }
    return 0;  // not reached for j below the level's task count
}

// Task t (< lvl[tmax]) of the interleaved order: its block and its tile within the block. One full warp.
__device__ __forceinline__ void level_locate(const uint32_t* prefix, int nseg, const uint32_t* lvl, uint32_t tmax,
                                             uint32_t t, int lane, int* sg, uint32_t* k) {
    uint32_t lo = 0, hi = tmax;  // lvl[lo] <= t < lvl[hi]
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (lvl[mid] <= t) lo = mid; else hi = mid;
    }
    *k = lo;
    *sg = level_pick(prefix, nseg, lo, t - lvl[lo], lane);
}

template <int KIND, int kStages, uint32_t kTile>
__global__ void __launch_bounds__(kCopyThreads) k_copy(const __grid_constant__ CopyArgs a) {
    static_assert(kStages <= 32, "stage phases live in one 32-bit mask");
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x;
    if (status_failed(a.ctl)) return;

    const int p = a.p;
    const int nseg = (KIND == COPY_BCAST) ? 1 : (KIND == COPY_ALLTOALL || KIND == COPY_ALLTOALLV) ? p * p : p;
    const int nseg_run = (KIND == COPY_ALLTOALLV && a.only_dst_plus1) ? p : nseg;  // segments this call copies
    unsigned char* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(kStages) * kTile);
    long long* sd = reinterpret_cast<long long*>(bars + kStages);
    long long* rd = sd + ((KIND == COPY_ALLTOALLV) ? p * p : 0);
    uint32_t* prefix = reinterpret_cast<uint32_t*>(rd + ((KIND == COPY_ALLTOALLV) ? p * p : 0));
    uint32_t* lvl = prefix + nseg + 1;  // a.level_cap + 1 entries

    if constexpr (KIND == COPY_ALLTOALLV) {
        const A2avPlan plan = a2av_plan_warp(a.counts, p, a.send_cap, a.recv_cap, sd, rd, a.recv_counts_out, a.ctl);
        if (!plan.ok) return;
    }
    {
    const int nseg = nseg_run;

    // tile counts per segment, then an inclusive scan into prefix[1..nseg]
    for (int s = lane; s < nseg; s += 32) {
        const SegDesc d = segment<KIND>(a, s, sd, rd);
        prefix[s + 1] = tile_count(reinterpret_cast<uintptr_t>(d.src), d.len, congruent(a, d), kTile);
    }
    __syncwarp();
    if (lane == 0) prefix[0] = 0;
    uint32_t carry = 0, tmax = 0, tmin = 0xFFFFFFFFu;
    for (int b = 0; b < nseg; b += 32) {
        const int s = b + lane;
        uint32_t v = (s < nseg) ? prefix[s + 1] : 0u;
        tmax = max(tmax, v);
        if (s < nseg) tmin = min(tmin, v);
#pragma unroll
        for (int dd = 1; dd < 32; dd <<= 1) {
            const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, v, dd);
            if (lane >= dd) v += o;
        }
        if (s < nseg) prefix[s + 1] = carry + v;
        carry += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
#pragma unroll
    for (int dd = 16; dd > 0; dd >>= 1) {
        tmax = max(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, dd));
        tmin = min(tmin, __shfl_xor_sync(0xFFFFFFFFu, tmin, dd));
    }
    __syncwarp();
    // Task order: segment-major, or interleaved (tile k of every segment before tile k+1 of any,
    // so all sources and destinations are streamed at once): through the level table when the
    // segments differ in size and it fits, else with empty slots skipped.
    const bool levels = a.order && tmin != tmax && tmax <= uint32_t(a.level_cap);
    if (levels) build_levels(prefix, nseg, tmax, lvl, lane);
    const uint32_t total = (a.order && !levels) ? tmax * uint32_t(nseg) : prefix[nseg];
    auto locate = [&](uint32_t t, int* sg, uint32_t* k) -> bool {
        if (!a.order) {
            *sg = find_segment(prefix, nseg, t);
            *k = t - prefix[*sg];
            return true;
        }
        if (levels) {
            level_locate(prefix, nseg, lvl, tmax, t, lane, sg, k);
            return true;
        }
        *sg = int(t % uint32_t(nseg));
        *k = t / uint32_t(nseg);
        return *k < prefix[*sg + 1] - prefix[*sg];
    };

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    __syncwarp();

    uint32_t phase = 0;  // bit s: parity of the next completion of stage s
    const uint64_t pol = a.l2_hint ? l2_evict_first_policy() : 0;
    bool failed = false;

    // A task is located once, when its load is issued, and handed to its consume through the stage's
    // slot. Tasks are claimed in increasing order, so the level pointer only moves forward.
    __shared__ int s_task_sg[kStages];
    __shared__ uint32_t s_task_ti[kStages];  // kNoTask: an empty slot of the interleaved order
    constexpr uint32_t kNoTask = 0xFFFFFFFFu;
    uint32_t lv = 0;
    auto issue = [&](uint32_t k, uint32_t t) {  // the k-th task of this CTA is task t
        int s = 0;
        uint32_t ti = 0;
        bool ok = true;
        if (levels) {
            while (lvl[lv + 1] <= t) ++lv;  // lv < tmax: t < lvl[tmax]
            s = level_pick(prefix, nseg, lv, t - lvl[lv], lane);
            ti = lv;
        } else {
            ok = locate(t, &s, &ti);
        }
        const int st = int(k % kStages);
        __syncwarp();
        if (lane == 0) {
            s_task_sg[st] = s;
            s_task_ti[st] = ok ? ti : kNoTask;
        }
        __syncwarp();
        if (!ok) return;
        const SegDesc d = segment<KIND>(a, s, sd, rd);
        const bool cong = congruent(a, d);
        const TileGeom g = tile_geom(reinterpret_cast<uintptr_t>(d.src), d.len, cong, ti, kTile);
        if (lane == 0 && g.bhi > g.blo) {
            mbar_arrive_expect_tx(&bars[st], uint32_t(g.bhi - g.blo));
            if (a.l2_hint == 1)
                bulk_g2s_hint(stages + size_t(st) * kTile, d.src + g.blo, uint32_t(g.bhi - g.blo), &bars[st], pol);
            else
                bulk_g2s(stages + size_t(st) * kTile, d.src + g.blo, uint32_t(g.bhi - g.blo), &bars[st]);
        }
    };

    auto consume = [&](uint32_t k) {
        const int s = s_task_sg[k % kStages];
        const uint32_t ti = s_task_ti[k % kStages];
        if (ti == kNoTask) return;
        const SegDesc d = segment<KIND>(a, s, sd, rd);
        const bool cong = congruent(a, d);
        const TileGeom g = tile_geom(reinterpret_cast<uintptr_t>(d.src), d.len, cong, ti, kTile);
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
                        if (dst == d.src) continue;
                        if (a.l2_hint) bulk_s2g_hint(dst + g.blo, src, bytes, pol);
                        else bulk_s2g(dst + g.blo, src, bytes);
                    }
                } else if (a.l2_hint) {
                    bulk_s2g_hint(d.dst + g.blo, src, bytes, pol);
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

    // Tasks are claimed one at a time, kStages - 1 ahead of the one being stored.
    uint32_t n_issued = 0;
    bool more = true;
    auto issue_next = [&]() {
        uint32_t t = 0;
        if (lane == 0) t = claim_task(a.ctl, &a.st->task_ctr, total);
        t = __shfl_sync(0xFFFFFFFFu, t, 0);
        if (t >= total) {
            more = false;
            return;
        }
        issue(n_issued, t);
        ++n_issued;
    };
    for (int k = 0; k < kStages - 1 && more; ++k) issue_next();
    for (uint32_t k = 0; k < n_issued && !failed; ++k) {
        if (more) {
            // the next task's stage was last used by task k-1, whose stores are the newest group
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            issue_next();
        }
        consume(k);
    }
    if (lane == 0) {
        bulk_wait_all();
        leave_tasks(&a.st->task_ctr, &a.st->done_ctr);
    }
    __syncwarp();
    }
}

// ---- load/store path -----------------------------------------------------------------------------
// Tasks of kLsuTask bytes of a segment, handed to 256-thread CTAs round-robin; a task is copied
// with 16-byte loads and stores (8 in flight per thread) where source and destination agree
// modulo 16, else with 2-byte accesses. Measured faster than the bulk-copy pipeline for 1:1
// copies (All-to-All(v)); the fan-out (Broadcast, AllGather) stays on bulk copies.
constexpr int kLsuThreads = 256;
constexpr int kLsuUnroll = 8;
constexpr uint32_t kLsuTask = 128 * 1024;

template <bool HINT>
__device__ __forceinline__ void cta_copy_bytes(const char* s, char* d, size_t bytes, uint64_t pol) {
    size_t head = bytes, body = 0;
    if (((reinterpret_cast<uintptr_t>(s) ^ reinterpret_cast<uintptr_t>(d)) & 15u) == 0) {
        head = (16 - (reinterpret_cast<uintptr_t>(s) & 15u)) & 15u;
        if (head > bytes) head = bytes;
        body = (bytes - head) & ~size_t(15);
    }
    for (size_t b = 2 * size_t(threadIdx.x); b < head; b += 2 * kLsuThreads)
        *reinterpret_cast<uint16_t*>(d + b) = *reinterpret_cast<const uint16_t*>(s + b);
    const Words<4>* vs = reinterpret_cast<const Words<4>*>(s + head);
    Words<4>* vd = reinterpret_cast<Words<4>*>(d + head);
    const size_t nv = body / 16;
    for (size_t v0 = threadIdx.x; v0 < nv; v0 += size_t(kLsuThreads) * kLsuUnroll) {
        Words<4> t[kLsuUnroll];
#pragma unroll
        for (int u = 0; u < kLsuUnroll; ++u) {
            const size_t v = v0 + size_t(u) * kLsuThreads;
            if (v < nv) t[u] = ld_pack<4, HINT>(vs + v, pol);
        }
#pragma unroll
        for (int u = 0; u < kLsuUnroll; ++u) {
            const size_t v = v0 + size_t(u) * kLsuThreads;
            if (v < nv) st_pack<4, HINT>(vd + v, t[u], pol);
        }
    }
    for (size_t b = head + body + 2 * size_t(threadIdx.x); b < bytes; b += 2 * kLsuThreads)
        *reinterpret_cast<uint16_t*>(d + b) = *reinterpret_cast<const uint16_t*>(s + b);
}

template <int KIND, bool HINT>
__global__ void __launch_bounds__(kLsuThreads, 2) k_copy_lsu(const __grid_constant__ CopyArgs a) {
    static_assert(KIND == COPY_ALLTOALL || KIND == COPY_ALLTOALLV, "1:1 segments only");
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_run;
    const int p = a.p;
    const int nseg_all = p * p;
    const int nseg = (KIND == COPY_ALLTOALLV && a.only_dst_plus1) ? p : nseg_all;  // segments this call copies
    long long* sd = reinterpret_cast<long long*>(smem);
    long long* rd = sd + ((KIND == COPY_ALLTOALLV) ? p * p : 0);
    uint32_t* prefix = reinterpret_cast<uint32_t*>(rd + ((KIND == COPY_ALLTOALLV) ? p * p : 0));
    uint32_t* lvl = prefix + nseg + 1;  // a.level_cap + 1 entries
    if (threadIdx.x == 0) s_run = !status_failed(a.ctl);
    __syncthreads();
    if (!s_run) return;
    if constexpr (KIND == COPY_ALLTOALLV) {
        if (threadIdx.x < 32) {
            const A2avPlan plan = a2av_plan_warp(a.counts, p, a.send_cap, a.recv_cap, sd, rd, a.recv_counts_out, a.ctl);
            if (threadIdx.x == 0) s_run = plan.ok;
        }
        __syncthreads();
        if (!s_run) return;
    }
    // tasks per segment and their prefix sums (warp 0), and the level table of the interleaved order
    __shared__ uint32_t s_tmax, s_levels;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        if (lane == 0) prefix[0] = 0;
        uint32_t carry = 0, tmax = 0, tmin = 0xFFFFFFFFu;
        for (int b = 0; b < nseg; b += 32) {
            const int sg = b + lane;
            uint32_t v = 0;
            if (sg < nseg) {
                const SegDesc d = segment<KIND>(a, sg, sd, rd);
                v = uint32_t((d.len + kLsuTask - 1) / kLsuTask);
                tmin = min(tmin, v);
            }
            tmax = max(tmax, v);
#pragma unroll
            for (int dd = 1; dd < 32; dd <<= 1) {
                const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, v, dd);
                if (lane >= dd) v += o;
            }
            if (sg < nseg) prefix[sg + 1] = carry + v;
            carry += __shfl_sync(0xFFFFFFFFu, v, 31);
        }
#pragma unroll
        for (int dd = 16; dd > 0; dd >>= 1) {
            tmax = max(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, dd));
            tmin = min(tmin, __shfl_xor_sync(0xFFFFFFFFu, tmin, dd));
        }
        __syncwarp();
        const bool levels = a.order && tmin != tmax && tmax <= uint32_t(a.level_cap);
        if (levels) build_levels(prefix, nseg, tmax, lvl, lane);
        if (lane == 0) {
            s_tmax = tmax;
            s_levels = levels;
        }
    }
    __syncthreads();
    const uint32_t tmax = s_tmax;
    const bool levels = s_levels != 0;
    const uint32_t total = (a.order && !levels) ? tmax * uint32_t(nseg) : prefix[nseg];
    uint64_t pol = 0;
    if constexpr (HINT) pol = l2_evict_first_policy();
    __shared__ uint32_t s_t;
    while (true) {
        __syncthreads();  // every thread has read the previous task number
        if (threadIdx.x == 0) s_t = claim_task(a.ctl, &a.st->task_ctr, total);
        __syncthreads();
        const uint32_t t = s_t;
        if (t >= total) break;
        int sg;
        uint32_t k;
        if (a.order && levels) {
            level_locate(prefix, nseg, lvl, tmax, t, threadIdx.x & 31, &sg, &k);  // every warp alike
        } else if (a.order) {
            sg = int(t % uint32_t(nseg));
            k = t / uint32_t(nseg);
            if (k >= prefix[sg + 1] - prefix[sg]) continue;
        } else {
            sg = find_segment(prefix, nseg, t);
            k = t - prefix[sg];
        }
        const SegDesc d = segment<KIND>(a, sg, sd, rd);
        const size_t lo = size_t(k) * kLsuTask;
        const size_t hi = min(lo + kLsuTask, d.len);
        cta_copy_bytes<HINT>(d.src + lo, d.dst + lo, hi - lo, pol);
    }
    if (threadIdx.x == 0) leave_tasks(&a.st->task_ctr, &a.st->done_ctr);
}

// ---- lean fan-out: Broadcast, AllGather (and the equal All-to-All) on 16-byte aligned buffers -------
// The fan-out pattern with nothing else on the critical path (the loop of the bulk fan-out probe):
// one lane issues everything; each segment (the root's buffer, or a rank's shard; for All-to-All
// block j of rank i, segment i * p + j) is cut into whole 32 KiB tiles, the last one shorter (a
// multiple of 16 bytes when the segment is); task t is tile t % per_seg of segment t / per_seg,
// claimed in order; a tile is loaded once and stored to every destination except the source itself
// (the in-place forms; All-to-All has one destination). Used when every buffer is 16-byte aligned
// and the segment a whole number of 16-byte units, so no tile needs a byte head or tail. LAG: before
// a stage is reloaded, wait only until the stores of the tile before the one just stored have read
// it (the stage being reloaded is that tile's), not for the latest tile's stores too.
constexpr uint32_t kFanTile = 32 * 1024;

template <int KIND, bool LAG, int STAGES>
__global__ void __launch_bounds__(32) k_fanout(const __grid_constant__ CopyArgs a) {
    static_assert(STAGES >= 2, "a stage is reloaded only after the tile before it was stored");
    static_assert(KIND == COPY_BCAST || KIND == COPY_ALLGATHER || KIND == COPY_ALLTOALL, "lean copy kinds only");
    extern __shared__ __align__(128) unsigned char stages[];
    __shared__ uint64_t bars[STAGES];
    __shared__ uint32_t s_task[STAGES];
    if (threadIdx.x != 0) return;
    if (status_failed(a.ctl)) return;
    const int p = a.p;
    const size_t seg_bytes = a.blk_elems * size_t(a.elem_bytes);
    const uint32_t per_seg = uint32_t((seg_bytes + kFanTile - 1) / kFanTile);
    const uint32_t total = per_seg * uint32_t(KIND == COPY_BCAST ? 1 : KIND == COPY_ALLTOALL ? p * p : p);
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
    const uint64_t pol = a.l2_hint ? l2_evict_first_policy() : 0;  // on the stores only
    auto source = [&](uint32_t t) -> const char* {
        const uint32_t q = t / per_seg;
        if constexpr (KIND == COPY_ALLTOALL)
            return static_cast<const char*>(a.ptrs.send[int(q) / p]) + size_t(q % uint32_t(p)) * seg_bytes +
                   size_t(t % per_seg) * kFanTile;
        return static_cast<const char*>(a.ptrs.send[KIND == COPY_BCAST ? a.root : int(q)]) +
               size_t(t % per_seg) * kFanTile;
    };
    auto tile_bytes = [&](uint32_t t) -> uint32_t {
        const size_t off = size_t(t % per_seg) * kFanTile;
        return uint32_t(min(size_t(kFanTile), seg_bytes - off));
    };
    uint32_t phase = 0, head = 0, tail = 0;
    bool more = true, failed = false;
    auto issue = [&]() {
        const uint32_t t = claim_task(a.ctl, &a.st->task_ctr, total);
        if (t >= total) {
            more = false;
            return;
        }
        const int st = int(head % STAGES);
        s_task[st] = t;
        mbar_arrive_expect_tx(&bars[st], tile_bytes(t));
        bulk_g2s(stages + size_t(st) * kFanTile, source(t), tile_bytes(t), &bars[st]);
        ++head;
    };
    while (more && head < STAGES - 1) issue();
    while (tail < head) {
        const int st = int(tail % STAGES);
        if (!mbar_wait_bounded(a.ctl, &bars[st], (phase >> st) & 1u, a.timeout_ns)) {
            failed = true;  // a load that never lands: stop issuing (the error is recorded)
            break;
        }
        phase ^= 1u << st;
        const uint32_t t = s_task[st];
        const char* src = source(t);
        const uint32_t bytes = tile_bytes(t);
        if constexpr (KIND == COPY_ALLTOALL) {
            const uint32_t q = t / per_seg;  // block q % p of rank q / p goes to rank q % p, block q / p
            char* dst = static_cast<char*>(a.ptrs.recv[int(q % uint32_t(p))]) + size_t(q / uint32_t(p)) * seg_bytes +
                        size_t(t % per_seg) * kFanTile;
            if (a.l2_hint) bulk_s2g_hint(dst, stages + size_t(st) * kFanTile, bytes, pol);
            else bulk_s2g(dst, stages + size_t(st) * kFanTile, bytes);
        } else {
            const size_t dst_off = (KIND == COPY_ALLGATHER ? size_t(t / per_seg) * seg_bytes : 0) +
                                   size_t(t % per_seg) * kFanTile;
            for (int r = 0; r < p; ++r) {
                char* dst = static_cast<char*>(a.ptrs.recv[r]) + dst_off;
                if (dst == src) continue;
                if (a.l2_hint) bulk_s2g_hint(dst, stages + size_t(st) * kFanTile, bytes, pol);
                else bulk_s2g(dst, stages + size_t(st) * kFanTile, bytes);
            }
        }
        bulk_commit();
        ++tail;
        if (more) {
            // the next load reuses the stage task tail-1 was stored from
            if constexpr (LAG) bulk_wait_read_but_last();
            else bulk_wait_read_all();
            issue();
        }
    }
    bulk_wait_all();
    if (!failed) leave_tasks(&a.st->task_ctr, &a.st->done_ctr);
}

// ---- one-pass copy: the equal All-to-All with 32-byte loads and stores --------------------------------
// A CTA per 32 KiB tile of a block (block j of rank i to rank j's block i, segment i * p + j, tiles in
// address order): the grid holds every tile and the hardware hands CTAs to SMs in order as they free
// up, as for the fused reduction's waves; each thread keeps its 4 x 32-byte loads in flight before its
// stores. Used when every buffer is 32-byte aligned and the block a whole number of 32-byte units.
constexpr int kPassThreads = 256;

template <int UNROLL>  // tile = 256 threads x UNROLL x 32 bytes
__global__ void __launch_bounds__(kPassThreads) k_a2a_pass(const __grid_constant__ CopyArgs a, uint32_t per_seg) {
    constexpr uint32_t kPassTile = uint32_t(kPassThreads) * UNROLL * 32;
    __shared__ int s_stop;
    if (threadIdx.x == 0) s_stop = status_failed(a.ctl);
    __syncthreads();
    if (s_stop) return;
    const size_t seg_bytes = a.blk_elems * size_t(a.elem_bytes);
    const uint32_t q = blockIdx.x / per_seg;
    const size_t off = size_t(blockIdx.x % per_seg) * kPassTile;
    const char* src = static_cast<const char*>(a.ptrs.send[int(q) / a.p]) + size_t(q % uint32_t(a.p)) * seg_bytes + off;
    char* dst = static_cast<char*>(a.ptrs.recv[int(q % uint32_t(a.p))]) + size_t(q / uint32_t(a.p)) * seg_bytes + off;
    const size_t nvec = min(size_t(kPassTile), seg_bytes - off) / 32;
    Words<8> v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
        const size_t k = threadIdx.x + size_t(u) * kPassThreads;
        if (k < nvec) v[u] = ld_stream_words<8>(src + k * 32);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
        const size_t k = threadIdx.x + size_t(u) * kPassThreads;
        if (k < nvec) st_words<8>(dst + k * 32, v[u]);
    }
}

static bool pass_ok(const CopyArgs& a) {
    if ((a.blk_elems * size_t(a.elem_bytes)) % 32 != 0) return false;
    for (int r = 0; r < a.p; ++r)
        if (reinterpret_cast<uintptr_t>(a.ptrs.send[r]) % 32 != 0 || reinterpret_cast<uintptr_t>(a.ptrs.recv[r]) % 32 != 0)
            return false;
    return true;
}

// The current device as one bit of a mask (0 for devices 63 and up, which set the attribute every launch).
static unsigned long long device_bit() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 63) return 0;
    return 1ull << dev;
}

// Level-table entries for the interleaved order (0 when the order is block after block).
static int level_cap(const CopyArgs& a) { return a.order ? kMaxLevels : 0; }

static size_t lsu_smem_bytes(int kind, int p, int levels) {
    size_t b = (kind == COPY_ALLTOALLV) ? 2 * size_t(p) * p * sizeof(long long) : 0;
    return b + (size_t(p) * p + 1) * sizeof(uint32_t) + (levels ? size_t(levels) + 1 : 0) * sizeof(uint32_t);
}

template <int KIND, bool HINT>
static cudaError_t launch_lsu_hint(const CopyArgs& a, int num_sms, cudaStream_t s) {
    static unsigned long long attr_set = 0;  // bit d: set on device d (a function attribute is per device)
    const unsigned long long bit = device_bit();
    if (!(attr_set & bit)) {
        cudaError_t e = cudaFuncSetAttribute(k_copy_lsu<KIND, HINT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(lsu_smem_bytes(KIND, kMaxRanks, kMaxLevels)));
        if (e != cudaSuccess) return e;
        attr_set |= bit;
    }
    CopyArgs b = a;
    b.level_cap = level_cap(a);
    k_copy_lsu<KIND, HINT><<<num_sms * 2, kLsuThreads, lsu_smem_bytes(KIND, a.p, b.level_cap), s>>>(b);
    return cudaGetLastError();
}

template <int KIND>
static cudaError_t launch_lsu(const CopyArgs& a, int num_sms, cudaStream_t s) {
    return a.l2_hint ? launch_lsu_hint<KIND, true>(a, num_sms, s) : launch_lsu_hint<KIND, false>(a, num_sms, s);
}

static size_t copy_smem_bytes(int kind, int p, int stages, uint32_t tile, int levels = 0) {
    const int nseg = (kind == COPY_BCAST) ? 1 : (kind == COPY_ALLTOALL || kind == COPY_ALLTOALLV) ? p * p : p;
    size_t b = size_t(stages) * tile + size_t(stages) * sizeof(uint64_t);
    if (kind == COPY_ALLTOALLV) b += 2 * size_t(p) * p * sizeof(long long);
    b += (size_t(nseg) + 1) * sizeof(uint32_t);
    if (levels) b += (size_t(levels) + 1) * sizeof(uint32_t);
    return (b + 127) & ~size_t(127);
}

static int max_smem_optin() {
    static int v = -1;
    if (v < 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            v = 48 * 1024;
    }
    return v;
}

static int max_smem_per_sm() {
    static int v = -1;
    if (v < 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
            v = 100 * 1024;
    }
    return v;
}

template <int KIND, int V>
static cudaError_t launch_shape(const CopyArgs& a, int num_sms, cudaStream_t s) {
    constexpr CopyShape sh = kCopyShapes[V];
    auto kernel = k_copy<KIND, sh.stages, sh.tile>;
    static unsigned long long attr_set = 0;  // bit d: set on device d
    const unsigned long long bit = device_bit();
    if (!(attr_set & bit)) {
        // the kernel's static shared memory (its stage slots) comes on top of the dynamic part
        const size_t want = std::min<size_t>(copy_smem_bytes(KIND, kMaxRanks, sh.stages, sh.tile, kMaxLevels),
                                             size_t(max_smem_optin()) - 1024);
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(want));
        if (e != cudaSuccess) return e;
        attr_set |= bit;
    }
    // the level table takes what the shape leaves of its share of the SM's shared memory (so the
    // shape's CTAs per SM still fit), up to kMaxLevels entries
    CopyArgs b = a;
    const size_t base = copy_smem_bytes(KIND, a.p, sh.stages, sh.tile);
    const long long budget = std::min<long long>(max_smem_optin() - 1024, max_smem_per_sm() / sh.ctas_per_sm - 2048);
    const long long room = (budget - static_cast<long long>(base) - 128) / 4 - 1;
    b.level_cap = int(std::max(0LL, std::min<long long>(level_cap(a), room)));
    kernel<<<num_sms * sh.ctas_per_sm, kCopyThreads, copy_smem_bytes(KIND, a.p, sh.stages, sh.tile, b.level_cap), s>>>(b);
    return cudaGetLastError();
}

template <int KIND>
static cudaError_t launch_kind(const CopyArgs& a, int num_sms, int variant, cudaStream_t s) {
    if (variant < 0 || variant >= kNumCopyShapes ||
        copy_smem_bytes(KIND, a.p, kCopyShapes[variant].stages, kCopyShapes[variant].tile) > size_t(max_smem_optin()) - 1024)
        variant = 0;  // the baseline shape fits every p
    switch (variant) {
        case 1: return launch_shape<KIND, 1>(a, num_sms, s);
        case 2: return launch_shape<KIND, 2>(a, num_sms, s);
        case 3: return launch_shape<KIND, 3>(a, num_sms, s);
        case 4: return launch_shape<KIND, 4>(a, num_sms, s);
        case 5: return launch_shape<KIND, 5>(a, num_sms, s);
        case 6: return launch_shape<KIND, 6>(a, num_sms, s);
        case 7: return launch_shape<KIND, 7>(a, num_sms, s);
        default: return launch_shape<KIND, 0>(a, num_sms, s);
    }
}

// Per-collective defaults, the fastest measured on B200 at the DP-bucket size (p = 8, 100 MiB per
// rank) with tasks claimed in order, each row charged with its own write-back. The general engine:
// 2 stages of 32 KiB with 3 CTAs per SM, block after block (All-to-All 0.257 ms against 0.345-0.405
// ms for the deeper 1-2 CTA shapes; All-to-Allv on the Zipf counts 0.266 ms against 0.276 on the
// load/store path and 0.282 in the interleaved order). On aligned buffers Broadcast and AllGather
// take the lean fan-out (0.160-0.161 ms against 0.166-0.167; lagged stage reuse 0.162-0.165), and
// the equal All-to-All the lean copy with lagged stage reuse, 4 stages, 1 CTA per SM (0.2546 ms
// against 0.2578 for the general engine and 0.2547-0.2556 for the other lagged shapes; on the MoE
// All-to-All, 8 x 8 MiB bf16 blocks per rank, 0.168-0.171 ms against 0.173; without the lag the
// lean copy takes 0.277 ms: a lane that waits for each tile's store to leave shared memory before
// reloading keeps too little in flight for a 1:1 copy).
constexpr int kVariantLsu = kNumCopyShapes;
constexpr int kVariantFan1 = kNumCopyShapes + 1;  // lean fan-out, 1 CTA per SM
constexpr int kVariantFan2 = kNumCopyShapes + 2;  // lean fan-out, 2 CTAs per SM
constexpr int kVariantFanLag1 = kNumCopyShapes + 3;  // lean, lagged stage reuse, 4 stages, 1 CTA per SM
constexpr int kVariantFanLag2 = kNumCopyShapes + 4;  // lean, lagged, 3 stages, 2 CTAs per SM
constexpr int kVariantFanLag3 = kNumCopyShapes + 5;  // lean, lagged, 6 stages, 1 CTA per SM
constexpr int kVariantFanLag4 = kNumCopyShapes + 6;  // lean, lagged, 2 stages, 3 CTAs per SM
constexpr int kVariantFan6 = kNumCopyShapes + 7;     // lean, 6 stages, 1 CTA per SM
constexpr int kVariantPass = kNumCopyShapes + 8;     // one-pass 32-byte load/store, 32 KiB per CTA (equal All-to-All)
constexpr int kVariantPass64 = kNumCopyShapes + 9;   // the same, 64 KiB per CTA
constexpr int kVariantPass16 = kNumCopyShapes + 10;  // the same, 16 KiB per CTA

void copy_defaults(int kind, int* variant, int* order) {
    *variant = (kind == COPY_BCAST || kind == COPY_ALLGATHER) ? kVariantFan1 : kind == COPY_ALLTOALL ? kVariantFanLag1 : 6;
    *order = 0;
}

// The lean fan-out path needs every touched buffer 16-byte aligned and whole 16-byte segments.
static bool fanout_ok(const CopyArgs& a) {
    if ((a.blk_elems * size_t(a.elem_bytes)) % 16 != 0) return false;
    for (int r = 0; r < a.p; ++r) {
        if (reinterpret_cast<uintptr_t>(a.ptrs.recv[r]) % 16 != 0) return false;
        if ((a.kind != COPY_BCAST || r == a.root) && reinterpret_cast<uintptr_t>(a.ptrs.send[r]) % 16 != 0)
            return false;
    }
    return true;
}

template <int KIND, bool LAG, int STAGES>
static cudaError_t launch_fanout(const CopyArgs& a, int num_sms, int ctas_per_sm, cudaStream_t s) {
    static unsigned long long attr_set = 0;  // bit d: set on device d
    const unsigned long long bit = device_bit();
    const size_t smem = size_t(STAGES) * kFanTile;
    if (!(attr_set & bit)) {
        cudaError_t e = cudaFuncSetAttribute(k_fanout<KIND, LAG, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        attr_set |= bit;
    }
    k_fanout<KIND, LAG, STAGES><<<num_sms * ctas_per_sm, 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <bool LAG, int STAGES>
static cudaError_t launch_lean(const CopyArgs& a, int num_sms, int cps, cudaStream_t s) {
    switch (a.kind) {
        case COPY_BCAST: return launch_fanout<COPY_BCAST, LAG, STAGES>(a, num_sms, cps, s);
        case COPY_ALLGATHER: return launch_fanout<COPY_ALLGATHER, LAG, STAGES>(a, num_sms, cps, s);
        default: return launch_fanout<COPY_ALLTOALL, LAG, STAGES>(a, num_sms, cps, s);
    }
}

// The L2 policy a copy takes by default: evict-first stores where the lean fan-out of Broadcast or
// AllGather runs (measured on B200, each row charged with its own write-back: 0.1607-0.1620 ms
// against 0.1634-0.1641 on the DP bucket; the stores leave fewer dirty lines behind), none elsewhere
// (the 1:1 All-to-All copy lost 1% with it).
int copy_path_l2_hint(const CopyArgs& a, int variant) {
    const bool fan = (a.kind == COPY_BCAST || a.kind == COPY_ALLGATHER) && variant >= kVariantFan1 &&
                     variant <= kVariantFan6 && fanout_ok(a);
    return fan ? 2 : 0;
}

cudaError_t launch_copy(const CopyArgs& a, int num_sms, int variant, cudaStream_t s) {
    if (variant >= kVariantPass && variant <= kVariantPass16) {
        if (a.kind == COPY_ALLTOALL && pass_ok(a)) {
            const int unroll = variant == kVariantPass ? 4 : variant == kVariantPass64 ? 8 : 2;
            const size_t tile = size_t(kPassThreads) * unroll * 32;
            const size_t seg_bytes = a.blk_elems * size_t(a.elem_bytes);
            const size_t per_seg = (seg_bytes + tile - 1) / tile;
            const size_t grid = per_seg * size_t(a.p) * size_t(a.p);
            if (grid == 0) return cudaSuccess;
            if (grid <= 0x7fffffffu) {
                if (unroll == 4) k_a2a_pass<4><<<unsigned(grid), kPassThreads, 0, s>>>(a, uint32_t(per_seg));
                else if (unroll == 8) k_a2a_pass<8><<<unsigned(grid), kPassThreads, 0, s>>>(a, uint32_t(per_seg));
                else k_a2a_pass<2><<<unsigned(grid), kPassThreads, 0, s>>>(a, uint32_t(per_seg));
                return cudaGetLastError();
            }
        }
        variant = 6;  // other collectives, or unaligned buffers: the general engine
    }
    if (variant >= kVariantFan1 && variant <= kVariantFan6) {
        const bool lean = (a.kind == COPY_BCAST || a.kind == COPY_ALLGATHER || a.kind == COPY_ALLTOALL) && fanout_ok(a);
        if (lean) {
            switch (variant) {
                case kVariantFan1: return launch_lean<false, 4>(a, num_sms, 1, s);
                case kVariantFan2: return launch_lean<false, 4>(a, num_sms, 2, s);
                case kVariantFanLag1: return launch_lean<true, 4>(a, num_sms, 1, s);
                case kVariantFanLag2: return launch_lean<true, 3>(a, num_sms, 2, s);
                case kVariantFanLag3: return launch_lean<true, 6>(a, num_sms, 1, s);
                case kVariantFanLag4: return launch_lean<true, 2>(a, num_sms, 3, s);
                default: return launch_lean<false, 6>(a, num_sms, 1, s);
            }
        }
        variant = 6;  // other collectives, or unaligned buffers: the general engine
    }
    if (variant == kVariantLsu) {
        if (a.kind == COPY_ALLTOALL) return launch_lsu<COPY_ALLTOALL>(a, num_sms, s);
        if (a.kind == COPY_ALLTOALLV) return launch_lsu<COPY_ALLTOALLV>(a, num_sms, s);
        variant = 5;  // the other collectives have no load/store variant
    }
    switch (a.kind) {
        case COPY_BCAST: return launch_kind<COPY_BCAST>(a, num_sms, variant, s);
        case COPY_ALLGATHER: return launch_kind<COPY_ALLGATHER>(a, num_sms, variant, s);
        case COPY_ALLTOALL: return launch_kind<COPY_ALLTOALL>(a, num_sms, variant, s);
        case COPY_ALLTOALLV: return launch_kind<COPY_ALLTOALLV>(a, num_sms, variant, s);
        case COPY_SCATTER: return launch_kind<COPY_SCATTER>(a, num_sms, variant, s);
        case COPY_GATHER: return launch_kind<COPY_GATHER>(a, num_sms, variant, s);
        default: return cudaErrorInvalidValue;
    }
}

int copy_num_variants() { return kNumCopyShapes + 11; }

}  // namespace simcomm
