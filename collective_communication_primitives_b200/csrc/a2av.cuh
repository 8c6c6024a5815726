// All-to-Allv planning: scan the shared count matrix into send and receive displacements.
//
// "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All", section
// "Ragged All-to-All：MoE 的真实输入通常不等长": c_ij elements go from source i to destination j;
// counts -> prefix-sum offsets -> payload exchange, and each pair's send and receive must agree
// (here they read the same matrix). Source i packs its blocks in destination order, destination j
// stores them in source order:
//   sdispl[i][j] = Σ_{j'<j} c[i][j'],   rdispl[i][j] = Σ_{i'<i} c[i'][j].
#pragma once

#include "common.cuh"

namespace simcomm {

__device__ __forceinline__ long long warp_inclusive_scan(long long v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        long long o = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += o;
    }
    return v;
}

__device__ __forceinline__ long long warp_max(long long v) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, d));
    return v;
}

struct A2avPlan {
    bool ok;
    long long max_count;  // largest single c_ij
};

// Run by one full warp. Writes sd[i*p+j] = sdispl, rd[i*p+j] = rdispl (shared memory), checks
// that no count is negative, that every row sum fits send_cap[i] and every column sum fits
// recv_cap[j]. The first CTA also writes the column sums to recv_counts_out (if given) and
// records COLL_ERR_OVERFLOW when a check fails. Every CTA reads the same counts, so every CTA
// reaches the same decision.
__device__ inline A2avPlan a2av_plan_warp(const long long* counts, int p, const long long* send_cap,
                                          const long long* recv_cap, long long* sd, long long* rd,
                                          long long* recv_counts_out, const Ctl& ctl) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
    long long mx = 0;
    // rows: send displacements
    for (int i = 0; i < p; ++i) {
        long long carry = 0;
        for (int j0 = 0; j0 < p; j0 += 32) {
            const int j = j0 + lane;
            const long long v = (j < p) ? counts[i * p + j] : 0;
            // a count above its row's capacity fails on its own, so with capacities at most 2^48
            // (checked on the host) no row or column sum below can wrap around
            if (v < 0 || v > send_cap[i]) bad = true;
            mx = max(mx, v);
            const long long incl = warp_inclusive_scan(v, lane);
            if (j < p) sd[i * p + j] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (carry > send_cap[i]) bad = true;
    }
    // columns: receive displacements
    for (int j = 0; j < p; ++j) {
        long long carry = 0;
        for (int i0 = 0; i0 < p; i0 += 32) {
            const int i = i0 + lane;
            const long long v = (i < p) ? counts[i * p + j] : 0;
            if (v > recv_cap[j]) bad = true;
            const long long incl = warp_inclusive_scan(v, lane);
            if (i < p) rd[i * p + j] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (carry > recv_cap[j]) bad = true;
        if (blockIdx.x == 0 && lane == 0 && recv_counts_out) recv_counts_out[j] = carry;
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    mx = warp_max(mx);
    if (bad && blockIdx.x == 0 && lane == 0) raise_status(ctl, COLL_ERR_OVERFLOW);
    __syncwarp();
    return A2avPlan{!bad, mx};
}

}  // namespace simcomm
