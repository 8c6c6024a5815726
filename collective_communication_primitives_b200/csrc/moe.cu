// MoE dispatch and combine: the steps on either side of the variable-split exchange, fused with it.
//
// Steps ("Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All",
// charlestar.github.io/2026/08/20/gpu-collective-communication, sections "Ragged All-to-All" and
// "Expert Parallel"): router output -> count assignments per destination -> exchange counts ->
// prefix-sum offsets -> pack/permute -> variable-split All-to-All -> expert compute -> reverse
// variable-split All-to-All -> unpermute and weighted combine (+ residual). One expert assignment
// (token t of rank i picked by slot s) is one row of H elements.
//
// Layout rules (our reading): expert e lives on rank e / (E/p); rank i's rows for rank j arrive in
// j's receive buffer after those of ranks 0..i-1, ordered by expert id, then token, then slot.
//
// Because all ranks share one memory, the pack and the exchange are one copy: every token row is
// read once and written straight into the k receive rows its assignments own; the reverse
// exchange, the unpermute and the weighted sum are likewise one pass that reads each token's k
// expert-output rows where the experts left them. The dispatch runs as one cooperative kernel,
// k_moe_dispatch_fused (below); the three kernels it fuses remain for devices without cooperative
// launches. Kernels:
//   k_moe_count   one CTA per (rank, tile of 256 assignments): validates expert ids, counts them per
//                 expert, and ranks every assignment among the tile's assignments of the same expert
//                 (warps in order; __match_any_sync groups equal experts inside a warp);
//   k_moe_scan    one CTA per rank: exclusive prefix of the tile counts over tiles, per expert; the
//                 last CTA to finish turns the per-rank totals into the count matrix c_ij, checks
//                 every destination's capacity and computes each (rank, expert)'s first receive row;
//   k_moe_dispatch_copy  one warp per token: the k destination rows (written to the routing map and
//                 kept in shared memory for the warp), then 16/32-byte streaming loads of the token
//                 row and k stores;
//   k_moe_combine one warp per token, tokens claimed in order: fp32 left fold in slot order
//                 (residual first), rounded once.
#include <algorithm>

#include "common.cuh"

namespace simcomm {

constexpr int kMoeThreads = kMoeTile;  // counting: one assignment per thread
constexpr int kScanThreads = 1024;
constexpr int kCopyThreads = 256;      // dispatch / combine: 8 warps, one token per warp at a time
constexpr int kCopyUnroll = 4;         // packs in flight per lane
constexpr int kCombineRegSlots = 2;    // combine: slots whose rows are loaded together with the residual

__device__ __forceinline__ bool cta_failed(const Ctl& ctl) {
    __shared__ int s_fail;
    if (threadIdx.x == 0) s_fail = status_failed(ctl);
    __syncthreads();
    const bool f = s_fail != 0;
    __syncthreads();
    return f;
}

// Programmatic dependent launch: the scan and the copy are launched while their predecessor in the
// stream still runs, and wait here (before touching anything it writes) until it has finished and
// its memory is visible; the predecessor lets them launch from its first instruction.
__device__ __forceinline__ void wait_for_predecessor() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- counting -----------------------------------------------------------------------------------

__global__ void __launch_bounds__(kMoeThreads) k_moe_count(const __grid_constant__ MoeArgs a) {
    extern __shared__ int s_cnt[];  // [E]
    allow_dependents();
    if (cta_failed(a.ctl)) return;
    const int i = blockIdx.y;
    const uint32_t tile = blockIdx.x;
    for (int e = threadIdx.x; e < a.E; e += kMoeThreads) s_cnt[e] = 0;
    __syncthreads();

    const size_t asg = size_t(tile) * kMoeTile + threadIdx.x;
    const bool valid = asg < a.A;
    int e = valid ? a.idx[i][asg] : -1;
    if (valid && (e < 0 || e >= a.E)) {
        raise_status(a.ctl, COLL_ERR_INVALID_ARG);
        e = -1;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int rank = 0;
    // warps take their turn in order so that ranks follow the assignment order
    for (int w = 0; w < kMoeThreads / 32; ++w) {
        if (warp == w) {
            const unsigned same = __match_any_sync(0xffffffffu, e);
            const int leader = __ffs(same) - 1;
            int first = 0;
            if (lane == leader && e >= 0) {
                first = s_cnt[e];
                s_cnt[e] = first + __popc(same);
            }
            first = __shfl_sync(0xffffffffu, first, leader);
            rank = first + __popc(same & ((1u << lane) - 1u));
        }
        __syncthreads();
    }
    if (valid) a.rank_in_tile[size_t(i) * a.A + asg] = rank;
    int32_t* hist = a.tile_hist + (size_t(i) * a.ntiles + tile) * a.E;
    for (int x = threadIdx.x; x < a.E; x += kMoeThreads) hist[x] = s_cnt[x];
}

// ---- prefix sums and the count matrix ------------------------------------------------------------

__device__ __forceinline__ int warp_incl_scan_i(int v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += o;
    }
    return v;
}

constexpr int kScanChunks = 4;        // tile counts of one expert a lane holds at once (128 tiles per pass)
constexpr int kScanSmemCnt = 4096;    // the last CTA stages the [p][E] totals in shared memory up to this many

__global__ void __launch_bounds__(kScanThreads) k_moe_scan(const __grid_constant__ MoeArgs a) {
    extern __shared__ int s_dyn[];  // [p][p] count matrix, then [p][E] totals (when they fit)
    __shared__ int s_last;
    wait_for_predecessor();
    allow_dependents();
    if (cta_failed(a.ctl)) return;
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kWarps = kScanThreads / 32;
    // per expert (a warp each, lanes over tiles): exclusive prefix of the tile counts of rank i, and the total
    for (int e = warp; e < a.E; e += kWarps) {
        int32_t* col = a.tile_hist + size_t(i) * a.ntiles * a.E + e;
        int run = 0;
        for (uint32_t t0 = 0; t0 < a.ntiles; t0 += 32 * kScanChunks) {
            int v[kScanChunks];
#pragma unroll
            for (int c = 0; c < kScanChunks; ++c) {
                const uint32_t t = t0 + uint32_t(c * 32 + lane);
                v[c] = t < a.ntiles ? col[size_t(t) * a.E] : 0;
            }
#pragma unroll
            for (int c = 0; c < kScanChunks; ++c) {
                const uint32_t t = t0 + uint32_t(c * 32 + lane);
                const int incl = warp_incl_scan_i(v[c], lane);
                if (t < a.ntiles) col[size_t(t) * a.E] = run + incl - v[c];
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (lane == 0) a.cnt[size_t(i) * a.E + e] = run;
    }
    // the last CTA to finish sees every rank's totals
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&a.st->moe_ctr, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int p = a.p;
    int* s_c = s_dyn;
    const bool staged = p * a.E <= kScanSmemCnt;
    int* s_cnt = s_dyn + p * p;
    if (staged)
        for (int x = threadIdx.x; x < p * a.E; x += kScanThreads) s_cnt[x] = __ldcg(a.cnt + x);
    __syncthreads();
    auto cnt_at = [&](int r, int x) -> int { return staged ? s_cnt[r * a.E + x] : __ldcg(a.cnt + size_t(r) * a.E + x); };
    for (int ij = threadIdx.x; ij < p * p; ij += kScanThreads) {  // c_ij: rows from rank i to rank j
        const int r = ij / p, j = ij % p;
        int sum = 0;
        for (int x = j * a.E_loc; x < (j + 1) * a.E_loc; ++x) sum += cnt_at(r, x);
        s_c[ij] = sum;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < p; j += kScanThreads) {  // rows arriving at rank j, against its capacity
        long long tot = 0;
        for (int r = 0; r < p; ++r) tot += s_c[r * p + j];
        if (size_t(tot) > a.cap_rows) raise_status(a.ctl, COLL_ERR_OVERFLOW);
        if (a.recv_counts_out) a.recv_counts_out[j] = tot;
    }
    for (int ie = threadIdx.x; ie < p * a.E; ie += kScanThreads) {  // first row of (rank i, expert e)
        const int r = ie / a.E, e = ie % a.E, j = e / a.E_loc;
        int b = 0;
        for (int q = 0; q < r; ++q) b += s_c[q * p + j];
        for (int x = j * a.E_loc; x < e; ++x) b += cnt_at(r, x);
        a.base[ie] = b;
        if (a.expert_counts_out) a.expert_counts_out[ie] = cnt_at(r, e);
    }
    if (threadIdx.x == 0) a.st->moe_ctr = 0;
}

// ---- dispatch: permute/pack fused with the exchange ---------------------------------------------

// Token batches: lane b*kslot + s holds slot s of the batch's b-th token (kslot = k rounded up to a
// power of two, so a batch holds 32/kslot tokens); the routes of a whole batch are looked up with one
// round of loads, then its tokens are copied one after another.
__device__ __forceinline__ int slot_width(int k) {
    int w = 1;
    while (w < k) w <<= 1;
    return w;
}

template <int W>
__global__ void __launch_bounds__(kCopyThreads) k_moe_dispatch_copy(const __grid_constant__ MoeArgs a) {
    __shared__ char* s_dst[kCopyThreads / 32][32];  // per warp: destination row of (batch token, slot)
    wait_for_predecessor();
    if (cta_failed(a.ctl)) return;
    const int i = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row_bytes = a.H * size_t(a.elem_bytes);
    const char* src = static_cast<const char*>(a.src[i]);
    char* const* dsts = s_dst[warp];
    const int kslot = slot_width(a.k), per_batch = 32 / kslot;
    const int my_b = lane / kslot, my_s = lane % kslot;
    // this warp's tokens: first, first + stride, first + 2 * stride, ...; a batch takes per_batch of them
    const size_t first = size_t(blockIdx.x) * (kCopyThreads / 32) + warp;
    const size_t stride = size_t(gridDim.x) * (kCopyThreads / 32);
    for (size_t t0 = first; t0 < a.T; t0 += stride * per_batch) {
        const size_t my_t = t0 + size_t(my_b) * stride;
        bool bad = false;
        if (my_s < a.k && my_t < a.T) {
            const size_t asg = my_t * a.k + my_s;
            const int e = a.idx[i][asg];
            const long long row = (long long)a.base[size_t(i) * a.E + e] +
                                  a.tile_hist[(size_t(i) * a.ntiles + asg / kMoeTile) * a.E + e] +
                                  a.rank_in_tile[size_t(i) * a.A + asg];
            bad = row < 0 || size_t(row) >= a.cap_rows;  // cannot happen after the capacity check
            if (bad) raise_status(a.ctl, COLL_ERR_INTERNAL);
            if (a.pos[i]) a.pos[i][asg] = bad ? -1 : int32_t(row);
            s_dst[warp][lane] = bad ? nullptr : static_cast<char*>(a.dst[e / a.E_loc]) + size_t(row) * row_bytes;
        }
        __syncwarp();
        if (!__any_sync(0xffffffffu, bad)) {
            for (int b = 0; b < per_batch; ++b) {
                const size_t t = t0 + size_t(b) * stride;
                if (t >= a.T) break;
                const char* s_row = src + t * row_bytes;
                char* const* d = dsts + b * kslot;
                if constexpr (W > 0) {
                    constexpr size_t kPack = size_t(W) * 4;
                    const size_t npk = row_bytes / kPack;
                    for (size_t c0 = lane; c0 < npk; c0 += 32 * kCopyUnroll) {
                        Words<W> v[kCopyUnroll];
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u)
                            if (c0 + u * 32 < npk) v[u] = ld_stream_words<W>(s_row + (c0 + u * 32) * kPack);
                        for (int s = 0; s < a.k; ++s) {
                            char* d_row = d[s];
#pragma unroll
                            for (int u = 0; u < kCopyUnroll; ++u)
                                if (c0 + u * 32 < npk) st_words<W>(d_row + (c0 + u * 32) * kPack, v[u]);
                        }
                    }
                } else {
                    // element-size-agnostic path: 2-byte units (every row is a whole number of them)
                    const size_t nu = row_bytes / 2;
                    for (size_t c0 = lane; c0 < nu; c0 += 32) {
                        const uint16_t v = *reinterpret_cast<const uint16_t*>(s_row + c0 * 2);
                        for (int s = 0; s < a.k; ++s) *reinterpret_cast<uint16_t*>(d[s] + c0 * 2) = v;
                    }
                }
            }
        }
        __syncwarp();  // the next batch rewrites this warp's destination rows
    }
}

// Bulk-copy variant: one warp per CTA; a task is one tile (at most kMoeTmaTile bytes) of one token
// row, loaded into shared memory by one bulk copy completing on an mbarrier and stored by one bulk
// copy per slot, with kMoeTmaStages tiles in flight. Needs rows of whole 16-byte units at 16-byte
// aligned bases (then every row start is aligned). No multicast form of any bulk copy is used.
constexpr int kMoeTmaStages = 8;
constexpr uint32_t kMoeTmaTile = 8192;
constexpr int kMoeTmaCtasPerSm = 3;

__global__ void __launch_bounds__(32) k_moe_dispatch_tma(const __grid_constant__ MoeArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ char* s_dst[kMoeMaxTopk];
    const int lane = threadIdx.x;
    wait_for_predecessor();
    if (status_failed(a.ctl)) return;  // one word read by every lane: the whole warp leaves together
    unsigned char* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(kMoeTmaStages) * kMoeTmaTile);
    const size_t row_bytes = a.H * size_t(a.elem_bytes);
    const size_t nq = (row_bytes + kMoeTmaTile - 1) / kMoeTmaTile;
    const size_t total = size_t(a.p) * a.T * nq;
    if (lane == 0) {
        for (int s = 0; s < kMoeTmaStages; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    __syncwarp();
    const size_t my_n = (total > blockIdx.x) ? (total - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    uint32_t phase = 0;  // bit s: parity of the next completion of stage s
    size_t issued = 0;   // tasks whose load has been issued
    struct Task { int i; size_t t, off; uint32_t bytes; };
    auto task_of = [&](size_t k) {
        const size_t u = blockIdx.x + k * gridDim.x;
        const size_t tok = u / nq;
        Task x;
        x.i = int(tok / a.T);
        x.t = tok % a.T;
        x.off = (u % nq) * kMoeTmaTile;
        x.bytes = uint32_t(min(size_t(kMoeTmaTile), row_bytes - x.off));
        return x;
    };
    auto issue = [&](size_t k) {
        issued = k + 1;
        if (lane != 0) return;
        const Task x = task_of(k);
        const int st = int(k % kMoeTmaStages);
        mbar_arrive_expect_tx(&bars[st], x.bytes);
        bulk_g2s(stages + size_t(st) * kMoeTmaTile, static_cast<const char*>(a.src[x.i]) + x.t * row_bytes + x.off,
                 x.bytes, &bars[st]);
    };
    auto wait_stage = [&](size_t k) -> bool {  // the load of task k has landed
        const int st = int(k % kMoeTmaStages);
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(a.ctl, &bars[st], (phase >> st) & 1u, a.timeout_ns);
        phase ^= (1u << st);
        return __shfl_sync(0xffffffffu, ok, 0);
    };
    // 0: done; 1: stop (a row out of range: nothing stored); 2: stop at once (a load never landed)
    auto consume = [&](size_t k) -> int {
        const Task x = task_of(k);
        bool bad = false;
        if (lane < a.k) {  // lane s: the receive row of slot s (written to the routing map once per row)
            const size_t asg = x.t * a.k + lane;
            const int e = a.idx[x.i][asg];
            const long long row = (long long)a.base[size_t(x.i) * a.E + e] +
                                  a.tile_hist[(size_t(x.i) * a.ntiles + asg / kMoeTile) * a.E + e] +
                                  a.rank_in_tile[size_t(x.i) * a.A + asg];
            bad = row < 0 || size_t(row) >= a.cap_rows;  // cannot happen after the capacity check
            if (x.off == 0 && a.pos[x.i]) a.pos[x.i][asg] = bad ? -1 : int32_t(row);
            s_dst[lane] = bad ? nullptr : static_cast<char*>(a.dst[e / a.E_loc]) + size_t(row) * row_bytes;
        }
        bad = __any_sync(0xffffffffu, bad);
        __syncwarp();
        if (!wait_stage(k)) return 2;
        if (bad) {
            if (lane == 0) raise_status(a.ctl, COLL_ERR_INTERNAL);
            return 1;
        }
        if (lane == 0) {
            fence_proxy_async_smem();
            const unsigned char* tile = stages + size_t(k % kMoeTmaStages) * kMoeTmaTile;
            for (int s = 0; s < a.k; ++s) bulk_s2g(s_dst[s] + x.off, tile, x.bytes);
            bulk_commit();
        }
        __syncwarp();  // s_dst is rewritten by the next task
        return 0;
    };
    const size_t pre = my_n < size_t(kMoeTmaStages - 1) ? my_n : size_t(kMoeTmaStages - 1);
    for (size_t k = 0; k < pre; ++k) issue(k);
    for (size_t k = 0; k < my_n; ++k) {
        const size_t kk = k + kMoeTmaStages - 1;
        if (kk < my_n) {
            // stage kk % kMoeTmaStages last held task k-1, whose stores are the newest group
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            issue(kk);
        }
        const int r = consume(k);
        if (r != 0) {
            if (r == 1)  // let the loads already issued land before the shared memory goes away
                for (size_t j = k + 1; j < issued; ++j) wait_stage(j);
            break;
        }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
}

// ---- fused dispatch: counting, prefix sums and the copy in one cooperative kernel -----------------
//
// Three kernels cost the dispatch ~23 us of launches and tiny serial phases before the copy starts
// (8 + 16 us under ncu on 8 x 8192 tokens). Here one cooperative launch (every CTA resident) runs
//   phase 1  counting: the k_moe_count work, a (rank, tile) per CTA pass, grid-strided; on the short
//            path (below) each tile's counts are also added into acc[i][e] (integer reductions:
//            exact in any order);
//   phase 2  (long path only) a warp per (rank, expert) column: exclusive prefix of the tile counts
//            over tiles, the total cnt[i][e] and c[i][j] += cnt[i][e];
//   phase 3  every CTA turns c into R[i][j] = sum over q < i of c[q][j] in shared memory (on the
//            short path after summing c[i][j] from acc) and checks every destination's capacity (the
//            same decision everywhere); base[i][e] = R[i][j] + the sum of cnt[i][.] over the block's
//            lower experts, built by every CTA in its shared memory when the table is small, else by
//            a warp per (rank, destination) block in global memory (with a third barrier);
//   phase 4  the copy: warps claim batches of consecutive token rows in order and copy each row with
//            32/16-byte loads and one store per slot. An assignment's row is base[i][e] + the count
//            of e in rank i's earlier tiles + its rank in its own tile: on the long path the middle
//            term is phase 2's prefix; on the short path the warp sums the earlier tiles' counts
//            itself, in the round trip that fetches the in-tile rank.
// with a bounded grid barrier between phases. The short path (base table in shared memory, at most
// kShortMaxTiles tiles per rank) has no phase 2 and no second barrier: the chain of dependent L2
// round trips before the copy starts is what a small dispatch costs. Data other CTAs wrote in this
// kernel is read through L2 (ld.global.cg): L1 is not coherent between SMs. acc is zeroed again by
// the call's last CTA (and by a reset after a failed call).
// Build-time knobs of the copy phase (measured on B200; the defaults are the fastest found).
#ifndef SIMCOMM_MOE_FUSED_UNROLL
#define SIMCOMM_MOE_FUSED_UNROLL 8   // packs in flight per lane
#endif
#ifndef SIMCOMM_MOE_FUSED_BATCH
#define SIMCOMM_MOE_FUSED_BATCH 1    // most token rows a warp claims at once (at most 32 / k rounded up)
#endif
constexpr int kFusedThreads = kMoeTile;  // a counting tile per CTA pass
constexpr int kFusedUnroll = SIMCOMM_MOE_FUSED_UNROLL;
constexpr int kWarpHistMaxE = 1024;      // per-warp counting histograms up to this many experts (32 KiB)
constexpr int kSmemBaseMax = 8192;       // every CTA keeps base[p][E] in shared memory up to this many entries
constexpr int kShortMaxTiles = 64;       // short path: tiles per rank (a lane sums at most two per lookup)
constexpr int kLookGroup = 4;            // short path: lookups whose earlier-tile counts load in one round trip

// Short path: the count of expert le in tiles [0, ltile) of rank li, for the lookup of every lane
// below nlook (lane = batch row x slot width + slot; lanes without a lookup pass ltile = 0). Warp-
// collective: the whole warp loads the earlier tiles' counts of kLookGroup lookups at once (at most
// two per lane, as ltile <= kShortMaxTiles) and reduces each.
__device__ __forceinline__ int earlier_tiles_count(const MoeArgs& a, int li, uint32_t ltile, int le, int nlook,
                                                   int lane) {
    int mine = 0;
    for (int q0 = 0; q0 < nlook; q0 += kLookGroup) {
        int v[kLookGroup][2];
#pragma unroll
        for (int q = 0; q < kLookGroup; ++q) {
            const int src = (q0 + q) & 31;
            const int qi = __shfl_sync(0xffffffffu, li, src);
            const uint32_t qt = q0 + q < nlook ? __shfl_sync(0xffffffffu, ltile, src) : 0u;
            const int qe = __shfl_sync(0xffffffffu, le, src);
            const int32_t* col = a.tile_hist + (size_t(qi) * a.E + qe) * a.ntiles;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t t = uint32_t(lane + 32 * r);
                v[q][r] = t < qt ? __ldcg(col + t) : 0;
            }
        }
#pragma unroll
        for (int q = 0; q < kLookGroup; ++q) {
            const int sum = int(__reduce_add_sync(0xffffffffu, unsigned(v[q][0] + v[q][1])));
            if (lane == q0 + q) mine = sum;
        }
    }
    return mine;
}

static size_t fused_smem_ints(int p, int E) {
    const size_t hist = E <= kWarpHistMaxE ? size_t(kFusedThreads / 32) * E : size_t(E);
    const size_t base = size_t(p) * E <= size_t(kSmemBaseMax) ? size_t(p) * E : 0;
    return size_t(p) * p + p + std::max(hist, base);
}

// The k-th grid barrier of a call (k = 1, 2, ...): every CTA adds 1 to moe_ctr with a release
// reduction (no return value, so no round trip) and polls moe_ctr until k rounds of arrivals are in,
// with a short sleep between polls. Measured on B200 with 296 CTAs: 1.4-1.8 us per barrier, against
// 1.8-2.3 us when each arrival is an atomic with a return and the last one releases a separate word
// (the serial L2 round trips set the cost; the kind of fence does not).
constexpr unsigned kBarrierPollSleepNs = 100;
__device__ __forceinline__ bool moe_grid_barrier(const MoeArgs& a, uint32_t k) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!(k == 1 && int(blockIdx.x) == a.skip_cta)) red_release_add_gpu(&a.st->moe_ctr, 1u);
        const uint32_t want = k * gridDim.x;
        bool ok = false;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 0; it < kMaxSpin; ++it) {
            if (ld_acquire_gpu(&a.st->moe_ctr) >= want) {
                ok = true;
                break;
            }
            __nanosleep(kBarrierPollSleepNs);
            if ((it & 255u) == 255u) {
                if (status_failed(a.ctl)) break;
                const uint64_t now = globaltimer_ns();
                if (now - t0 > a.timeout_ns) {
                    raise_status(a.ctl, COLL_ERR_TIMEOUT);
                    break;
                }
                if (abort_requested(a.ctl, now)) {
                    raise_status(a.ctl, COLL_ERR_ABORTED);
                    break;
                }
            }
        }
        if (!ok && !status_failed(a.ctl)) raise_status(a.ctl, COLL_ERR_TIMEOUT);
        s_ok = ok && !status_failed(a.ctl);
    }
    __syncthreads();
    return s_ok != 0;
}

template <int W>
__global__ void __launch_bounds__(kFusedThreads, 2) k_moe_dispatch_fused(const __grid_constant__ MoeArgs a) {
    // dynamic shared memory: [p][p] c -> R, [p] column totals, then a region used first for the
    // counting histograms ([8][E] per-warp counts when E <= kWarpHistMaxE, else [E]) and then, when
    // p * E <= kSmemBaseMax, for the first rows base[p][E]
    extern __shared__ int s_dyn[];
    __shared__ char* s_dst[kFusedThreads / 32][32];
    __shared__ int s_flag;
    if (cta_failed(a.ctl)) return;
    const int p = a.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* s_c = s_dyn;
    int* s_tot = s_c + p * p;
    int* s_cnt = s_tot + p;
    const bool warp_hist = a.E <= kWarpHistMaxE;
    const int hist_ints = warp_hist ? (kFusedThreads / 32) * a.E : a.E;
    const bool smem_base = p * a.E <= kSmemBaseMax;
    const bool short_path = smem_base && a.ntiles <= uint32_t(kShortMaxTiles) && a.acc != nullptr;
    int* s_base = s_cnt;

    // ---- phase 1: counting ----
    if (blockIdx.x == 0 && !short_path)
        for (int x = threadIdx.x; x < p * p; x += kFusedThreads) a.cmat[x] = 0;
    const uint32_t ntask = uint32_t(p) * a.ntiles;
    // this thread's expert id in the CTA's g-th tile (-1 past the end); the next tile's id is loaded
    // before the current tile is counted, so its latency overlaps the counting
    auto load_id = [&](uint32_t g) -> int {
        if (g >= ntask) return -1;
        const size_t asg = size_t(g % a.ntiles) * kMoeTile + threadIdx.x;
        return asg < a.A ? a.idx[g / a.ntiles][asg] : -1;
    };
    int e_next = load_id(blockIdx.x);
    for (uint32_t g = blockIdx.x; g < ntask; g += gridDim.x) {
        const int i = int(g / a.ntiles);
        const uint32_t tile = g % a.ntiles;
        int e = e_next;
        e_next = load_id(g + gridDim.x);
        __syncthreads();  // the previous tile's histogram has been written out
        for (int x = threadIdx.x; x < hist_ints; x += kFusedThreads) s_cnt[x] = 0;
        __syncthreads();
        const size_t asg = size_t(tile) * kMoeTile + threadIdx.x;
        const bool valid = asg < a.A;
        if (valid && (e < 0 || e >= a.E)) {
            raise_status(a.ctl, COLL_ERR_INVALID_ARG);
            e = -1;
        }
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int leader = __ffs(same) - 1;
        const int below = __popc(same & ((1u << lane) - 1u));  // same-expert assignments before it in the warp
        int rank = 0;
        int32_t* hist = a.tile_hist + size_t(i) * a.E * a.ntiles + tile;  // expert x at hist[x * ntiles]
        if (warp_hist) {
            // every warp counts its own experts, then an assignment's rank adds the counts of the
            // warps before it: no turn-taking
            if (lane == leader && e >= 0) s_cnt[warp * a.E + e] = __popc(same);
            __syncthreads();
            if (e >= 0) {
                for (int w = 0; w < warp; ++w) rank += s_cnt[w * a.E + e];
                rank += below;
            }
            for (int x = threadIdx.x; x < a.E; x += kFusedThreads) {
                int t = 0;
#pragma unroll
                for (int w = 0; w < kFusedThreads / 32; ++w) t += s_cnt[w * a.E + x];
                hist[size_t(x) * a.ntiles] = t;
                if (short_path && t != 0) atomicAdd(a.acc + size_t(i) * a.E + x, t);
            }
        } else {
            for (int w = 0; w < kFusedThreads / 32; ++w) {  // warps in order: ranks follow assignment order
                if (warp == w) {
                    int first = 0;
                    if (lane == leader && e >= 0) {
                        first = s_cnt[e];
                        s_cnt[e] = first + __popc(same);
                    }
                    rank = __shfl_sync(0xffffffffu, first, leader) + below;
                }
                __syncthreads();
            }
            for (int x = threadIdx.x; x < a.E; x += kFusedThreads) {
                hist[size_t(x) * a.ntiles] = s_cnt[x];
                if (short_path && s_cnt[x] != 0) atomicAdd(a.acc + size_t(i) * a.E + x, s_cnt[x]);
            }
        }
        if (valid) a.rank_in_tile[size_t(i) * a.A + asg] = rank;
    }
    if (!moe_grid_barrier(a, 1)) return;

    // ---- phase 2 (long path): per (rank, expert) column, prefix over tiles, totals ----
    const uint32_t nwarps = gridDim.x * (kFusedThreads / 32);
    const uint32_t gw = blockIdx.x * (kFusedThreads / 32) + uint32_t(warp);
    for (uint32_t col = gw; !short_path && col < uint32_t(p) * uint32_t(a.E); col += nwarps) {
        const int i = int(col / uint32_t(a.E)), e = int(col % uint32_t(a.E));
        int32_t* colp = a.tile_hist + (size_t(i) * a.E + e) * a.ntiles;
        int run = 0;
        for (uint32_t t0 = 0; t0 < a.ntiles; t0 += 32 * kScanChunks) {
            int v[kScanChunks];
#pragma unroll
            for (int c = 0; c < kScanChunks; ++c) {
                const uint32_t t = t0 + uint32_t(c * 32 + lane);
                v[c] = t < a.ntiles ? __ldcg(colp + t) : 0;
            }
#pragma unroll
            for (int c = 0; c < kScanChunks; ++c) {
                const uint32_t t = t0 + uint32_t(c * 32 + lane);
                const int incl = warp_incl_scan_i(v[c], lane);
                if (t < a.ntiles) colp[t] = run + incl - v[c];
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (lane == 0) {
            a.cnt[size_t(i) * a.E + e] = run;
            atomicAdd(&a.cmat[i * p + e / a.E_loc], run);
            if (a.expert_counts_out) a.expert_counts_out[size_t(i) * a.E + e] = run;
        }
    }
    if (!short_path && !moe_grid_barrier(a, 2)) return;

    // ---- phase 3: R = exclusive column prefix of c, capacity check, first rows ----
    if (short_path) {
        // the totals from acc, then c[i][j] = the sum of cnt[i][e] over rank j's experts
        for (int x = threadIdx.x; x < p * a.E; x += kFusedThreads) s_base[x] = __ldcg(a.acc + x);
        if (threadIdx.x == 0) s_flag = 0;
        __syncthreads();
        if (blockIdx.x == 0 && a.expert_counts_out)
            for (int x = threadIdx.x; x < p * a.E; x += kFusedThreads) a.expert_counts_out[x] = s_base[x];
        for (int blk = threadIdx.x; blk < p * p; blk += kFusedThreads) {
            const int i = blk / p, j = blk % p;
            int t = 0;
            for (int e = j * a.E_loc; e < (j + 1) * a.E_loc; ++e) t += s_base[i * a.E + e];
            s_c[blk] = t;
        }
    } else {
        for (int x = threadIdx.x; x < p * p; x += kFusedThreads) s_c[x] = __ldcg(a.cmat + x);
        if (smem_base)  // the totals too, in the same round trip
            for (int x = threadIdx.x; x < p * a.E; x += kFusedThreads) s_base[x] = __ldcg(a.cnt + x);
        if (threadIdx.x == 0) s_flag = 0;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < p; j += kFusedThreads) {
        int run = 0;
        for (int q = 0; q < p; ++q) {
            const int v = s_c[q * p + j];
            s_c[q * p + j] = run;
            run += v;
        }
        s_tot[j] = run;
        if (size_t(run) > a.cap_rows) atomicOr(&s_flag, 1);
        if (blockIdx.x == 0 && a.recv_counts_out) a.recv_counts_out[j] = run;
    }
    __syncthreads();
    if (s_flag) {  // every CTA computed the same totals: nobody copies anything
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(a.ctl, COLL_ERR_OVERFLOW);
        return;
    }
    if (smem_base) {
        // every CTA builds the whole table in its shared memory: no third barrier
        for (int blk = threadIdx.x; blk < p * p; blk += kFusedThreads) {  // (rank, destination) blocks
            const int i = blk / p, j = blk % p;
            int run = s_c[i * p + j];
            for (int e = j * a.E_loc; e < (j + 1) * a.E_loc; ++e) {
                const int v = s_base[i * a.E + e];
                s_base[i * a.E + e] = run;
                run += v;
            }
        }
        __syncthreads();
    } else {
        for (uint32_t blk = gw; blk < uint32_t(p) * uint32_t(p); blk += nwarps) {
            const int i = int(blk / uint32_t(p)), j = int(blk % uint32_t(p));
            int run = s_c[i * p + j];
            for (int e0 = j * a.E_loc; e0 < (j + 1) * a.E_loc; e0 += 32) {
                const int e = e0 + lane;
                const int v = e < (j + 1) * a.E_loc ? __ldcg(a.cnt + size_t(i) * a.E + e) : 0;
                const int incl = warp_incl_scan_i(v, lane);
                if (e < (j + 1) * a.E_loc) a.base[size_t(i) * a.E + e] = run + incl - v;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (!moe_grid_barrier(a, 3)) return;
    }

    // ---- phase 4: the copy, batches of consecutive token rows claimed in order ----
    const size_t row_bytes = a.H * size_t(a.elem_bytes);
    const int kslot = slot_width(a.k), per_batch = min(32 / kslot, SIMCOMM_MOE_FUSED_BATCH);
    const int my_b = lane / kslot, my_s = lane % kslot;
    const unsigned long long rows = (unsigned long long)p * a.T;
    while (true) {
        unsigned long long u0 = 0;
        if (lane == 0) u0 = status_failed(a.ctl) ? rows : atomicAdd(&a.st->moe_task, (unsigned long long)per_batch);
        u0 = __shfl_sync(0xffffffffu, u0, 0);
        if (u0 >= rows) break;
        const unsigned long long my_u = u0 + unsigned(my_b);
        const bool look = my_s < a.k && my_b < per_batch && my_u < rows;
        int i = 0, e = 0, in_tile = 0;
        uint32_t tile = 0;
        size_t asg = 0;
        if (look) {
            i = int(my_u / a.T);
            asg = size_t(my_u % a.T) * a.k + my_s;
            e = a.idx[i][asg];
            tile = uint32_t(asg / kMoeTile);
            in_tile = __ldcg(a.rank_in_tile + size_t(i) * a.A + asg);
        }
        const int earlier = short_path ? earlier_tiles_count(a, i, tile, e, per_batch * kslot, lane)
                            : look    ? __ldcg(a.tile_hist + (size_t(i) * a.E + e) * a.ntiles + tile)
                                      : 0;
        bool bad = false;
        if (look) {
            const int first = smem_base ? s_base[i * a.E + e] : __ldcg(a.base + size_t(i) * a.E + e);
            const long long row = (long long)first + earlier + in_tile;
            bad = row < 0 || size_t(row) >= a.cap_rows;  // cannot happen after the capacity check
            if (bad) raise_status(a.ctl, COLL_ERR_INTERNAL);
            if (a.pos[i]) a.pos[i][asg] = bad ? -1 : int32_t(row);
            const int owner = e / a.E_loc;
            const bool mine = a.view_rank < 0 || owner == a.view_rank;  // a rank view copies to itself only
            s_dst[warp][lane] = bad || !mine ? nullptr : static_cast<char*>(a.dst[owner]) + size_t(row) * row_bytes;
        }
        __syncwarp();
        if (!__any_sync(0xffffffffu, bad)) {
            for (int b = 0; b < per_batch; ++b) {
                const unsigned long long u = u0 + unsigned(b);
                if (u >= rows) break;
                const char* s_row = static_cast<const char*>(a.src[int(u / a.T)]) + size_t(u % a.T) * row_bytes;
                char* const* d = s_dst[warp] + b * kslot;
                if (a.view_rank >= 0) {  // a row none of whose slots goes to this rank is not read
                    bool any = false;
                    for (int sl = 0; sl < a.k; ++sl) any = any || d[sl] != nullptr;
                    if (!any) continue;
                }
                if constexpr (W > 0) {
                    constexpr size_t kPack = size_t(W) * 4;
                    const size_t npk = row_bytes / kPack;
                    for (size_t c0 = lane; c0 < npk; c0 += 32 * kFusedUnroll) {
                        Words<W> v[kFusedUnroll];
#pragma unroll
                        for (int q = 0; q < kFusedUnroll; ++q)
                            if (c0 + q * 32 < npk) v[q] = ld_stream_words<W>(s_row + (c0 + q * 32) * kPack);
                        for (int sl = 0; sl < a.k; ++sl) {
                            char* d_row = d[sl];
                            if (a.view_rank >= 0 && !d_row) continue;
#pragma unroll
                            for (int q = 0; q < kFusedUnroll; ++q)
                                if (c0 + q * 32 < npk) st_words<W>(d_row + (c0 + q * 32) * kPack, v[q]);
                        }
                    }
                } else {
                    const size_t nu = row_bytes / 2;  // 2-byte units (every row is a whole number of them)
                    for (size_t c0 = lane; c0 < nu; c0 += 32) {
                        const uint16_t v = *reinterpret_cast<const uint16_t*>(s_row + c0 * 2);
                        for (int sl = 0; sl < a.k; ++sl)
                            if (d[sl]) *reinterpret_cast<uint16_t*>(d[sl] + c0 * 2) = v;
                    }
                }
            }
        }
        __syncwarp();  // the next batch rewrites this warp's destination rows
    }
    // the last CTA out clears the call's counters and totals (every CTA has read them by now)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_flag = atomicAdd(&a.st->done_ctr, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_flag) {
        if (short_path)
            for (int x = threadIdx.x; x < p * a.E; x += kFusedThreads) a.acc[x] = 0;
        if (threadIdx.x == 0) {
            a.st->moe_task = 0;
            a.st->moe_ctr = 0;
            a.st->done_ctr = 0;
        }
        __threadfence();
    }
}

// ---- combine: reverse exchange + unpermute + weighted sum ---------------------------------------

template <int DT>
__device__ __forceinline__ void unpack4(const uint4& v, float (&x)[16 / Elem<DT>::kBytes]) {
    if constexpr (DT == COLL_BF16) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            x[2 * q] = bf16_bits_to_float(w[q] & 0xffffu);
            x[2 * q + 1] = bf16_bits_to_float(w[q] >> 16);
        }
    } else {
        x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
    }
}

template <int DT>
__device__ __forceinline__ uint4 pack4(const float (&x)[16 / Elem<DT>::kBytes]) {
    if constexpr (DT == COLL_BF16) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = uint32_t(float_to_bf16_bits(x[2 * q])) | (uint32_t(float_to_bf16_bits(x[2 * q + 1])) << 16);
        return make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
    }
}

template <int DT>
__device__ __forceinline__ float load_f(const void* base, size_t e) {
    if constexpr (DT == COLL_BF16) return bf16_bits_to_float(static_cast<const uint16_t*>(base)[e]);
    else return static_cast<const float*>(base)[e];
}

template <int DT>
__device__ __forceinline__ void store_f(void* base, size_t e, float v) {
    if constexpr (DT == COLL_BF16) static_cast<uint16_t*>(base)[e] = float_to_bf16_bits(v);
    else static_cast<float*>(base)[e] = v;
}

// VEC: 16-byte packs (every row start 16-byte aligned); otherwise one element per lane.
template <int DT, bool VEC>
__global__ void __launch_bounds__(kCopyThreads) k_moe_combine(const __grid_constant__ MoeArgs a) {
    constexpr int L = 16 / Elem<DT>::kBytes;
    __shared__ const char* s_y[kCopyThreads / 32][kMoeMaxTopk];  // per warp: the token's k expert-output rows
    __shared__ float s_w[kCopyThreads / 32][kMoeMaxTopk];        // and their gate weights
    if (cta_failed(a.ctl)) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t d = size_t(Elem<DT>::kBytes);
    const char* const* ys = s_y[warp];
    const float* ws = s_w[warp];
    // warps claim tokens in order (rank-major) from a counter; a rank view combines its own tokens
    const unsigned long long total = (a.view_rank >= 0 ? 1ull : (unsigned long long)a.p) * a.T;
    while (true) {
        unsigned long long u = 0;
        if (lane == 0) u = status_failed(a.ctl) ? total : atomicAdd(&a.st->comb_task, 1ull);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= total) break;
        const int i = a.view_rank >= 0 ? a.view_rank : int(u / a.T);
        const size_t t = size_t(u % a.T);
        bool bad = false;
        if (lane < a.k) {
            const size_t asg = t * a.k + lane;
            const int e = a.idx[i][asg];
            const int r = a.pos[i][asg];
            bad = e < 0 || e >= a.E || r < 0 || size_t(r) >= a.cap_rows;
            s_y[warp][lane] = bad ? nullptr : static_cast<const char*>(a.src[e / a.E_loc]) + size_t(r) * a.H * d;
            s_w[warp][lane] = a.w[i][asg];
        }
        __syncwarp();
        if (__any_sync(0xffffffffu, bad)) {
            if (lane == 0) raise_status(a.ctl, COLL_ERR_INVALID_ARG);
            __syncwarp();
            continue;
        }
        char* o_row = static_cast<char*>(a.dst[i]) + t * a.H * d;
        const char* r_row = a.has_res ? static_cast<const char*>(a.res[i]) + t * a.H * d : nullptr;
        if constexpr (VEC) {
            const size_t npk = a.H / L;
            if (a.k <= kCombineRegSlots) {
                // every load of a chunk (the residual and up to kCombineRegSlots rows) in flight at once
                for (size_t c0 = lane; c0 < npk; c0 += 32 * kCopyUnroll) {
                    uint4 rv[kCopyUnroll], yv[kCombineRegSlots][kCopyUnroll];
#pragma unroll
                    for (int u = 0; u < kCopyUnroll; ++u) {
                        if (c0 + u * 32 >= npk) continue;
                        if (r_row) rv[u] = ld_stream_v4(r_row + (c0 + u * 32) * 16);
#pragma unroll
                        for (int s = 0; s < kCombineRegSlots; ++s)
                            if (s < a.k) yv[s][u] = ld_stream_v4(ys[s] + (c0 + u * 32) * 16);
                    }
#pragma unroll
                    for (int u = 0; u < kCopyUnroll; ++u) {
                        if (c0 + u * 32 >= npk) continue;
                        float acc[L], y[L];
                        int s0 = 0;
                        if (r_row) {
                            unpack4<DT>(rv[u], acc);
                        } else {
                            unpack4<DT>(yv[0][u], acc);
#pragma unroll
                            for (int l = 0; l < L; ++l) acc[l] = ws[0] * acc[l];
                            s0 = 1;
                        }
#pragma unroll
                        for (int s = 0; s < kCombineRegSlots; ++s) {
                            if (s < s0 || s >= a.k) continue;
                            unpack4<DT>(yv[s][u], y);
                            const float w = ws[s];
#pragma unroll
                            for (int l = 0; l < L; ++l) acc[l] = acc[l] + w * y[l];
                        }
                        st_v4(o_row + (c0 + u * 32) * 16, pack4<DT>(acc));
                    }
                }
            } else {
                for (size_t c0 = lane; c0 < npk; c0 += 32 * kCopyUnroll) {
                    float acc[kCopyUnroll][L];
                    int s0 = 0;
                    if (r_row) {
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u)
                            if (c0 + u * 32 < npk) unpack4<DT>(ld_stream_v4(r_row + (c0 + u * 32) * 16), acc[u]);
                    } else {
                        const float w0 = ws[0];
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u) {
                            if (c0 + u * 32 < npk) {
                                unpack4<DT>(ld_stream_v4(ys[0] + (c0 + u * 32) * 16), acc[u]);
#pragma unroll
                                for (int l = 0; l < L; ++l) acc[u][l] = w0 * acc[u][l];
                            }
                        }
                        s0 = 1;
                    }
                    for (int s = s0; s < a.k; ++s) {
                        const char* y_row = ys[s];
                        const float w = ws[s];
                        uint4 v[kCopyUnroll];
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u)
                            if (c0 + u * 32 < npk) v[u] = ld_stream_v4(y_row + (c0 + u * 32) * 16);
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u) {
                            if (c0 + u * 32 < npk) {
                                float y[L];
                                unpack4<DT>(v[u], y);
#pragma unroll
                                for (int l = 0; l < L; ++l) acc[u][l] = acc[u][l] + w * y[l];
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kCopyUnroll; ++u)
                        if (c0 + u * 32 < npk) st_v4(o_row + (c0 + u * 32) * 16, pack4<DT>(acc[u]));
                }
            }
        } else {
            for (size_t h = lane; h < a.H; h += 32) {
                float acc;
                int s0 = 0;
                if (r_row) {
                    acc = load_f<DT>(r_row, h);
                } else {
                    acc = ws[0] * load_f<DT>(ys[0], h);
                    s0 = 1;
                }
                for (int s = s0; s < a.k; ++s) acc = acc + ws[s] * load_f<DT>(ys[s], h);
                store_f<DT>(o_row, h, acc);
            }
        }
        __syncwarp();  // the next token rewrites this warp's rows and weights
    }
    // the last CTA out resets the counter for the next call
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&a.st->comb_done, 1u) == gridDim.x * gridDim.y - 1) {
            a.st->comb_task = 0;
            a.st->comb_done = 0;
            __threadfence();
        }
    }
}

// ---- launch --------------------------------------------------------------------------------------

// One wave: the CTAs that fit on the device at once (resident_per_sm from the kernel's occupancy),
// split evenly over the ranks, each striding over its rank's tokens.
static dim3 token_grid(const MoeArgs& a, int num_sms, int resident_per_sm) {
    const size_t warps_per_cta = kCopyThreads / 32;
    const size_t want = (a.T + warps_per_cta - 1) / warps_per_cta;
    const size_t ranks = a.view_rank >= 0 ? 1 : size_t(a.p);  // a rank view: its own rank's tokens only
    const size_t per_rank = std::max<size_t>(1, size_t(num_sms) * size_t(std::max(resident_per_sm, 1)) / ranks);
    return dim3(unsigned(std::max<size_t>(1, std::min(want, per_rank))), unsigned(ranks), 1u);
}

template <typename K>
static int resident_per_sm(K kernel) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kCopyThreads, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

// A launch that may begin while the stream's previous kernel still runs (the kernel waits for it
// with griddepcontrol.wait before reading what it wrote).
static cudaError_t launch_after(void (*kernel)(MoeArgs), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                const MoeArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// The fused dispatch on a cooperative launch: as many CTAs as are resident at once (needed by its
// grid barriers). Returns cudaErrorNotSupported when the device cannot launch cooperatively.
template <int W>
static cudaError_t launch_fused(const MoeArgs& a, int num_sms, cudaStream_t s) {
    auto kernel = k_moe_dispatch_fused<W>;
    const size_t smem = fused_smem_ints(a.p, a.E) * sizeof(int);
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kFusedThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorNotSupported;
    dim3 grid(unsigned(num_sms * per_sm)), block(kFusedThreads);
    MoeArgs b = a;
    void* args[] = {&b};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kernel), grid, block, args, smem, s);
    return e != cudaSuccess ? e : cudaGetLastError();
}

static bool cooperative_ok() {
    static int v = -1;
    if (v < 0) {
        int dev = 0, ok = 0;
        v = (cudaGetDevice(&dev) == cudaSuccess &&
             cudaDeviceGetAttribute(&ok, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && ok) ? 1 : 0;
    }
    return v == 1;
}

cudaError_t launch_moe_dispatch(const MoeArgs& a, int num_sms, cudaStream_t s, int* kernels_launched) {
    *kernels_launched = 0;
    if (a.view_rank >= 0 && !(a.fused && cooperative_ok())) return cudaErrorNotSupported;  // views: fused only
    if (a.fused && cooperative_ok()) {
        *kernels_launched = 1;
        const size_t row_bytes = a.H * size_t(a.elem_bytes);
        bool al32 = row_bytes % 32 == 0, al16 = row_bytes % 16 == 0;
        for (int r = 0; r < a.p; ++r) {
            const uintptr_t x = reinterpret_cast<uintptr_t>(a.src[r]), y = reinterpret_cast<uintptr_t>(a.dst[r]);
            al32 = al32 && x % 32 == 0 && y % 32 == 0;
            al16 = al16 && x % 16 == 0 && y % 16 == 0;
        }
        if (al32) return launch_fused<8>(a, num_sms, s);
        if (al16) return launch_fused<4>(a, num_sms, s);
        return launch_fused<0>(a, num_sms, s);
    }
    *kernels_launched = 3;
    const size_t smem_count = size_t(a.E) * sizeof(int);
    if (smem_count > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_moe_count, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_count));
        if (e != cudaSuccess) return e;
    }
    k_moe_count<<<dim3(a.ntiles, unsigned(a.p), 1u), kMoeThreads, smem_count, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem_scan = (size_t(a.p) * a.p + (size_t(a.p) * a.E <= size_t(kScanSmemCnt) ? size_t(a.p) * a.E : 0)) *
                             sizeof(int);
    if ((e = launch_after(k_moe_scan, dim3(unsigned(a.p)), dim3(kScanThreads), smem_scan, s, a)) != cudaSuccess)
        return e;
    // bulk copies when chosen and every row start is 16-byte aligned; else 32-byte packs when every
    // row start is 32-byte aligned, else 16-byte, else 2-byte units
    const size_t row_bytes = a.H * size_t(a.elem_bytes);
    bool al32 = row_bytes % 32 == 0, al16 = row_bytes % 16 == 0;
    for (int r = 0; r < a.p; ++r) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a.src[r]), y = reinterpret_cast<uintptr_t>(a.dst[r]);
        al32 = al32 && x % 32 == 0 && y % 32 == 0;
        al16 = al16 && x % 16 == 0 && y % 16 == 0;
    }
    if (a.tma && al16) {
        const size_t smem = size_t(kMoeTmaStages) * kMoeTmaTile + kMoeTmaStages * sizeof(uint64_t);
        e = cudaFuncSetAttribute(k_moe_dispatch_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        const size_t tasks = size_t(a.p) * a.T * ((row_bytes + kMoeTmaTile - 1) / kMoeTmaTile);
        const size_t ctas = std::min(tasks, size_t(num_sms) * kMoeTmaCtasPerSm);
        return launch_after(k_moe_dispatch_tma, dim3(unsigned(std::max<size_t>(ctas, 1))), dim3(32), smem, s, a);
    }
    auto copy = [&](auto kernel) {
        return launch_after(kernel, token_grid(a, num_sms, resident_per_sm(kernel)), dim3(kCopyThreads), 0, s, a);
    };
    if (al32) return copy(k_moe_dispatch_copy<8>);
    if (al16) return copy(k_moe_dispatch_copy<4>);
    return copy(k_moe_dispatch_copy<0>);
}

cudaError_t launch_moe_combine(const MoeArgs& a, int dtype, int num_sms, cudaStream_t s) {
    const size_t row_bytes = a.H * size_t(a.elem_bytes);
    bool vec = row_bytes % 16 == 0;
    for (int r = 0; r < a.p; ++r) {
        vec = vec && reinterpret_cast<uintptr_t>(a.src[r]) % 16 == 0 && reinterpret_cast<uintptr_t>(a.dst[r]) % 16 == 0;
        if (a.has_res) vec = vec && reinterpret_cast<uintptr_t>(a.res[r]) % 16 == 0;
    }
    // one wave of resident CTAs whose warps claim tokens in order
    auto go = [&](auto kernel) {
        const size_t warps_per_cta = kCopyThreads / 32;
        const size_t tokens = a.T * size_t(a.view_rank >= 0 ? 1 : a.p);
        const size_t want = (tokens + warps_per_cta - 1) / warps_per_cta;
        const size_t wave = size_t(num_sms) * size_t(resident_per_sm(kernel));
        kernel<<<unsigned(std::max<size_t>(1, std::min(want, wave))), kCopyThreads, 0, s>>>(a);
    };
    if (dtype == COLL_BF16) {
        if (vec) go(k_moe_combine<COLL_BF16, true>);
        else go(k_moe_combine<COLL_BF16, false>);
    } else if (dtype == COLL_FP32) {
        if (vec) go(k_moe_combine<COLL_FP32, true>);
        else go(k_moe_combine<COLL_FP32, false>);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace simcomm
