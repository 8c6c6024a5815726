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
    uint32_t task_ctr;  // ring, tree, butterfly executors and the copy kernels: next task to claim
    uint32_t done_ctr;  // the same kernels: CTAs that left the task loop (the last one resets both)
    uint32_t moe_ctr;   // MoE dispatch: scan blocks finished, or the fused kernel's grid-barrier arrivals
                        // (zero between calls)
    uint32_t step_ctr[32];  // butterfly executor: finished tasks per step (zero between calls)
    unsigned long long abort_clock;  // global time of the last read of the host abort word
    unsigned long long moe_task;     // fused MoE dispatch: next token row to claim (zero between calls)
    unsigned long long comb_task;    // MoE combine: next token to claim (zero between calls)
    uint32_t comb_done;              // MoE combine: CTAs that left the token loop (the last one resets both)
};

// What a kernel needs to report errors and notice an abort.
struct Ctl {
    uint32_t* status;                  // &DevState::status
    volatile uint32_t* host_status;    // device alias of a host-mapped word the host polls
    volatile const uint32_t* abort_flag;  // device alias of the host-mapped abort flag
    unsigned long long* abort_clock;      // &DevState::abort_clock: rations the reads of abort_flag
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
    int level_cap;                     // order 1: entries of the shared-memory level table (0 = none)
    int l2_hint;                       // 1: evict-first L2 policy on the bulk/streaming copies
    const long long* counts;           // ALLTOALLV: device [p][p]
    long long* recv_counts_out;        // ALLTOALLV: device [p] or null
    long long send_cap[kMaxRanks];     // ALLTOALLV: elements per send buffer
    long long recv_cap[kMaxRanks];     // ALLTOALLV: elements per recv buffer
    uint64_t timeout_ns;
    DevState* st;                      // task counters (dynamic distribution)
    int only_dst_plus1;                // ALLTOALLV of a rank view: 1 + the one destination it copies, 0 = all
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
    int skip_rank;           // fault injection: this rank's tasks are never counted (-1 = off)
    uint64_t timeout_ns;
    char* stage;             // RD: two partial buffers per rank; HD: one
    size_t stage_stride;
    DevState* st;
    Ctl ctl;
};

// ---- tree executor: single and double binary tree AllReduce -------------------------------------

constexpr int kMaxTreeSteps = 16;
struct TreeArgs {
    RankPtrs ptrs;
    int p;
    int ntrees;              // 1: tree A over [0, n); 2: tree A over [0, half), tree B over [half, n)
    int vec;                 // 1: 16-byte packs (every range start 16-byte aligned)
    size_t n, half;
    size_t chunk;            // elements of one pipelined chunk
    size_t tile;             // elements one CTA task moves
    uint32_t ntile;          // tasks per chunk
    uint32_t nch[2];         // chunks of each tree's range
    uint32_t nchmax;
    uint32_t nsteps;         // reduce levels (deepest first), then broadcast levels (root side first)
    uint32_t step_kind[kMaxTreeSteps];   // 0 reduce, 1 broadcast
    uint32_t step_first[kMaxTreeSteps];  // first heap position of the step
    uint32_t step_count[kMaxTreeSteps];  // positions in the step
    uint32_t start[kMaxTreeSteps + 1];   // first task of each step
    uint32_t epoch;
    float scale;
    int skip_rank;           // fault injection: this rank never signals (-1 = off)
    uint64_t timeout_ns;
    char* stage;             // partials, one buffer per rank
    size_t stage_stride;
    unsigned long long* flags;  // [phase][tree][position][nchmax]: (epoch << 32) | finished tiles
    DevState* st;
    Ctl ctl;
};

// ---- low-latency (LL) ring AllReduce --------------------------------------------------------------

enum LLKind { LL_RING = 0, LL_RD = 1, LL_RING_RS = 2, LL_RING_AG = 3, LL_TREE = 4 };
struct LLArgs {
    RankPtrs ptrs;
    int kind;                // LL_RING (AllReduce), LL_RING_RS, LL_RING_AG, LL_RD or LL_TREE
    int ept;                 // LL_RD: elements per thread, held in registers (1, 2, 4 or 8)
    int p;
    int G;                   // CTAs per rank
    int GA;                  // LL_TREE: CTAs per rank on tree A's elements (the other G - GA carry tree B's)
    size_t n;                // elements per rank
    size_t seg;              // ring segment, ceil(n / p); LL_TREE: elements of tree A (n for the single tree)
    uint32_t nslots;         // receive slots per rank: one per step that crosses a hop (ring 2p - 3, RD log2 p)
    uint32_t tag;            // this call's tag of slot 0 (slot q carries tag + q)
    float scale;
    int skip_rank;           // fault injection: this rank never sends (-1 = off)
    uint64_t timeout_ns;
    unsigned long long* ll;  // ring [p][nslots][seg], RD and tree [p][nslots][n] words: (tag << 32) | 32 data bits
    Ctl ctl;
};

// ---- MoE dispatch and combine ------------------------------------------------------------------

constexpr int kMoeTile = 256;         // assignments per counting tile (one per thread)
constexpr int kMoeMaxExperts = 4096;  // the counting tile keeps one int per expert in shared memory
constexpr int kMoeMaxTopk = 32;       // one lane per slot of a token

struct MoeArgs {
    const void* src[kMaxRanks];      // dispatch: token rows x_i [T][H]; combine: expert outputs y_j [rows][H]
    const int32_t* idx[kMaxRanks];   // router output [T][k] expert ids
    int32_t* pos[kMaxRanks];         // [T][k] row of each assignment at its owner (dispatch writes it, or null)
    void* dst[kMaxRanks];            // dispatch: receive buffers [cap_rows][H]; combine: outputs [T][H]
    const float* w[kMaxRanks];       // combine: gate weights [T][k]
    const void* res[kMaxRanks];      // combine: residual [T][H] (has_res)
    int p, k, E, E_loc;
    int elem_bytes;
    int has_res;
    size_t T, H;                     // tokens per rank, elements per row
    size_t A;                        // assignments per rank, T*k
    size_t cap_rows;                 // rows of every receive buffer (dispatch) / expert-output buffer (combine)
    uint32_t ntiles;                 // counting tiles per rank, ceil(A / kMoeTile)
    int32_t* tile_hist;              // [p][ntiles][E] per-tile expert counts, then exclusive prefix over tiles
                                     // (the fused dispatch lays it out [p][E][ntiles])
    int32_t* rank_in_tile;           // [p][A] rank of an assignment among its tile's same-expert ones
    int32_t* cnt;                    // [p][E] assignments from rank i to expert e
    int32_t* base;                   // [p][E] first receive row of (rank i, expert e) at the expert's owner
    int32_t* cmat;                   // fused dispatch: [p][p] rows from rank i to rank j
    int32_t* acc;                    // fused dispatch: [p][E] totals summed during counting (zero between calls)
    long long* expert_counts_out;    // [p][E] or null
    long long* recv_counts_out;      // [p] or null
    int tma;                         // dispatch copy: 1 bulk copies through shared memory, 0 loads/stores
    int view_rank;                   // a rank view: the one rank whose outputs the call writes (-1: every rank)
    int skip_cta;                    // fault injection: this CTA of the fused dispatch never arrives at its
                                     // first grid barrier (-1 = off)
    int fused;                       // dispatch: 1 one cooperative kernel (counting, sums and copy), 0 three
                                     // kernels (the copy chosen by tma)
    uint64_t timeout_ns;
    DevState* st;
    Ctl ctl;
};

// ---- HBM access-pattern probes (not collectives) --------------------------------------------------
enum ProbeKind { PROBE_LOAD = 0, PROBE_STORE = 1, PROBE_COPY = 2, PROBE_BULK_STORE = 3, PROBE_BULK_FANOUT = 4 };
constexpr int kProbeFanCopies = 8;  // PROBE_BULK_FANOUT writes this many copies of src

// Launchers (each returns the launch error; grid sizes are decided inside).
cudaError_t launch_butterfly(const ButterflyArgs& a, int dtype, int op, int ctas, cudaStream_t s);
cudaError_t launch_direct_reduce(const DirectReduceArgs& a, int dtype, int op, int num_sms, cudaStream_t s);
cudaError_t launch_copy(const CopyArgs& a, int num_sms, int variant, cudaStream_t s);
int copy_num_variants();
void copy_defaults(int kind, int* variant, int* order);
int copy_path_l2_hint(const CopyArgs& a, int variant);  // the l2_hint a copy takes by default (option -1)
cudaError_t launch_ring(const RingArgs& a, int dtype, int op, int ctas, cudaStream_t s);
int ring_max_ctas(int num_sms);
cudaError_t launch_ring_ll(const LLArgs& a, int dtype, int op, cudaStream_t s);
int ring_ll_max_ctas(int num_sms);
cudaError_t launch_tree(const TreeArgs& a, int dtype, int op, int ctas, cudaStream_t s);
cudaError_t launch_moe_dispatch(const MoeArgs& a, int num_sms, cudaStream_t s, int* kernels_launched);
cudaError_t launch_moe_combine(const MoeArgs& a, int dtype, int num_sms, cudaStream_t s);
cudaError_t launch_probe(int kind, void* dst, const void* src, size_t bytes, int ctas_per_sm, int num_sms,
                         cudaStream_t s);

}  // namespace simcomm
