// Internal structures shared by the host API (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "simcomm.h"

namespace simcomm {

constexpr int kMaxRanks = SIM_COMM_MAX_RANKS;

// Device scratch header of a communicator (device memory, zero-initialised).
struct DevState {
    uint32_t status;    // first asynchronous error (coll_status_t), 0 = OK
    uint32_t task_ctr;  // ring / butterfly executor: next task to claim
    uint32_t done_ctr;  // ring / butterfly executor: CTAs that left the task loop
    uint32_t pad;
    uint32_t step_ctr[32];  // butterfly executor: finished tasks per step (zero between calls)
};

// What a kernel needs to report errors and notice an abort.
struct Ctl {
    uint32_t* status;                  // &DevState::status
    volatile uint32_t* host_status;    // device alias of a host-mapped word the host polls
    volatile const uint32_t* abort_flag;  // device alias of the host-mapped abort flag
};

struct RankPtrs {
    const void* send[kMaxRanks];
    void* recv[kMaxRanks];
};

// ---- direct fused reduction (AllReduce / Reduce / ReduceScatter) ---------------------------------
enum DirectMode { MODE_ALLREDUCE = 0, MODE_REDUCE = 1, MODE_REDUCE_SCATTER = 2 };

struct DirectReduceArgs {
    RankPtrs ptrs;
    int p;
    int mode;
    int root;
    int vec;           // 2: 32-byte packs, 1: 16-byte packs, 0: element-wise
    size_t n;          // per-rank full element count
    size_t seg;        // ReduceScatter: elements per owner (n / p); otherwise n
    float scale;       // AVG: 1/p; otherwise 1
    int ctas_per_sm;   // grid = SMs x this (capped by the work)
    int l2_hint;       // 1: evict-first L2 policy on the streaming loads and stores
    Ctl ctl;
};

// ---- copy engine (Broadcast / AllGather / All-to-All / All-to-Allv) ------------------------------
enum CopyKind { COPY_BCAST = 0, COPY_ALLGATHER = 1, COPY_ALLTOALL = 2, COPY_ALLTOALLV = 3, COPY_SCATTER = 4,
                COPY_GATHER = 5 };

struct CopyArgs {
    RankPtrs ptrs;
    int p;
    int kind;
    int root;
    int elem_bytes;
    size_t blk_elems;                  // BCAST: n; ALLGATHER, ALLTOALL, SCATTER, GATHER: block n/p
    int order;                         // tile order: 0 segment-major, 1 interleaved over segments
    int l2_hint;                       // 1: evict-first L2 policy on the bulk/streaming copies
    const long long* counts;           // ALLTOALLV: device [p][p]
    long long* recv_counts_out;        // ALLTOALLV: device [p] or null
    long long send_cap[kMaxRanks];     // ALLTOALLV: elements per send buffer
    long long recv_cap[kMaxRanks];     // ALLTOALLV: elements per recv buffer
    uint64_t timeout_ns;
    Ctl ctl;
};

// ---- ring executor -----------------------------------------------------------------------------
enum RingKind {
    RING_ALLREDUCE = 0, RING_REDUCE_SCATTER = 1, RING_ALLGATHER = 2, RING_REDUCE = 3,
    RING_BCAST = 4, RING_ALLTOALL = 5, RING_ALLTOALLV = 6
};

struct RingArgs {
    RankPtrs ptrs;
    int p;
    int kind;
    int root;
    int vec;                 // 1: vectorised reduce hops (all offsets 16-byte aligned)
    int elem_bytes;          // bytes per element
    size_t n;                // per-rank full element count
    size_t seg;              // elements of one segment (the unit a step moves)
    size_t chunk;            // elements of one pipelined chunk
    size_t tile;             // elements one CTA task moves (a chunk is split into ntile of them)
    uint32_t ntile;          // CTA tasks per chunk
    uint32_t nch;            // chunks per segment (ALLTOALLV: computed on the device)
    uint32_t nsteps;         // steps of the schedule
    uint32_t ranks_per_step; // p for ring steps, 1 for the Reduce/Broadcast chains
    uint32_t epoch;          // flags equal to epoch mean "done in this call"
    float scale;
    int skip_rank;           // fault injection: this rank never signals (-1 = off)
    uint64_t timeout_ns;
    char* stage;             // partial buffers, one per rank
    size_t stage_stride;     // bytes between ranks' partial buffers
    unsigned long long* flags;  // [nsteps][ranks_per_step][nch]: (epoch << 32) | finished tiles
    DevState* st;
    const long long* counts; // ALLTOALLV
    long long* recv_counts_out;
    long long send_cap[kMaxRanks];
    long long recv_cap[kMaxRanks];
    Ctl ctl;
};

// ---- butterfly executor: recursive doubling and halving-doubling AllReduce ---------------------
enum ButterflyKind { BFLY_RD = 0, BFLY_HD = 1 };
constexpr int kMaxBflySteps = 16;

struct ButterflyArgs {
    RankPtrs ptrs;
    int p;
    int kind;
    int log2p;
    int vec;                 // 1: 16-byte hops (every range start 16-byte aligned)
    size_t n;
    size_t seg;              // block size (ceil(n/p)), HD only
    size_t tile;             // elements per CTA task
    uint32_t nsteps;
    uint32_t ntile[kMaxBflySteps];   // tasks per rank at each step
    uint32_t start[kMaxBflySteps + 1];  // first task of each step
    float scale;
    uint64_t timeout_ns;
    char* stage;             // RD: two partial buffers per rank; HD: one
    size_t stage_stride;
    DevState* st;
    Ctl ctl;
};

// Launchers (each returns the launch error; grid sizes are decided inside).
cudaError_t launch_butterfly(const ButterflyArgs& a, int dtype, int op, int ctas, cudaStream_t s);
cudaError_t launch_direct_reduce(const DirectReduceArgs& a, int dtype, int op, int num_sms, cudaStream_t s);
cudaError_t launch_copy(const CopyArgs& a, int num_sms, int variant, cudaStream_t s);
int copy_num_variants();
void copy_defaults(int kind, int* variant, int* order);
cudaError_t launch_ring(const RingArgs& a, int dtype, int op, int ctas, cudaStream_t s);
int ring_max_ctas(int num_sms);

}  // namespace simcomm
