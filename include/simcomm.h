/*
 * simcomm.h — C ABI of the simulated-communicator collectives on one B200.
 *
 * A communicator of p logical ranks lives inside one GPU: rank r owns its own device buffers,
 * and a collective reads and writes all p ranks' buffers in HBM. Every call only enqueues work
 * on the caller's CUDA stream and returns; completion is observed through that stream.
 *
 * Pages cited (title, then section):
 *   [Atlas]  "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives)
 *   [Primer] "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All"
 *            (charlestar.github.io/2026/08/20/gpu-collective-communication)
 *   [Eight]  "详解分布式训练8大集合通信原语：从Send/Recv到All2All" (bjdmk.com.cn/news/4699717)
 *
 * Common conventions
 *   - n is the per-rank FULL buffer element count ([Primer] "先统一通信量的记号": B is the full
 *     logical tensor): the AllReduce input/output, the ReduceScatter input, the AllGather output,
 *     the All-to-All send buffer. ReduceScatter outputs, AllGather inputs and All-to-All blocks
 *     hold n/p elements.
 *   - A root is a rank index in [0, p), not a device number ([Atlas] §0, §1.1).
 *   - bufs.send and bufs.recv are HOST arrays of p DEVICE pointers (rank order). The arrays are
 *     read during the call only; the device buffers are owned by the caller and must stay alive,
 *     and unchanged by other work, until the stream reaches the end of the collective
 *     ([Primer] "CUDA Stream：API 返回不代表结果可被 Host 或其他 Stream 读取").
 *   - Buffers are contiguous and element-aligned. 16-byte-aligned buffers whose block sizes are
 *     multiples of 16 bytes take the vector/bulk-copy paths; anything else takes a slower
 *     element-wise path with the same results.
 *   - bf16 data is reduced in fp32 and rounded once (round to nearest, ties to even) to bf16.
 *     AVG is SUM times 1/p in fp32, applied before that rounding. int32 SUM wraps around
 *     (two's complement). MIN/MAX keep the earlier rank on ties. AVG is not defined for int32.
 *   - In place is allowed only in the forms of [Primer] "In-place 不是“任意让输入输出指向同一地址”":
 *     AllReduce send[r] == recv[r]; AllGather send[r] == recv[r] + r·(n/p); ReduceScatter
 *     recv[r] == send[r] + r·(n/p); Reduce/Broadcast the root's send == recv. Any other overlap
 *     between an output and any buffer is rejected with COLL_ERR_INVALID_ARG. All-to-All and
 *     All-to-Allv are never in place.
 *   - One communicator runs one collective at a time: calls on different streams must be ordered
 *     by the caller (the communicator's scratch is shared between calls).
 *   - Calls on a communicator may be captured into a CUDA graph (stream capture) and the graph
 *     replayed any number of times, with eager calls of the same communicator in between. A
 *     captured call's scratch must already exist: make the same call once before capturing; a call
 *     that would have to grow the scratch under capture returns COLL_ERR_UNSUPPORTED and enqueues
 *     nothing. The schedules whose signals carry a per-call epoch or tag (ring, tree, LL) add a
 *     memset node that clears the flags or slots they use, so each replay starts clean. Once a call
 *     has been captured, scratch that a later (larger) call replaces stays allocated until
 *     sim_comm_destroy, since a graph may still use it; destroy the communicator only after its
 *     graphs.
 *
 * Errors
 *   - Synchronous (returned, nothing enqueued): COLL_ERR_INVALID_ARG (null handle or pointer, bad
 *     root/dtype/op/algo, n not divisible by p where required, illegal aliasing), COLL_ERR_UNSUPPORTED,
 *     COLL_ERR_CUDA (a CUDA call failed; sim_comm_last_error() has the message), and the sticky
 *     asynchronous error of an earlier call, if the host has already seen it.
 *   - Asynchronous (set on the device, read with sim_comm_get_async_error): COLL_ERR_TIMEOUT (a
 *     bounded device wait ran out: a ring, tree or butterfly step for its predecessor, an LL word,
 *     a bulk copy), COLL_ERR_ABORTED (sim_comm_abort was called while such a wait was running),
 *     COLL_ERR_OVERFLOW (an All-to-Allv count or an MoE dispatch exceeds a capacity; nothing is
 *     copied), COLL_ERR_INVALID_ARG (an MoE expert id or routing-map entry out of range),
 *     COLL_ERR_INTERNAL (an invariant check failed). Collectives are not transactions: after an
 *     asynchronous error the outputs of the failed call are unspecified, and later calls do no
 *     work until sim_comm_reset ([Primer] "Collective 的故障语义不是事务").
 */
#ifndef SIMCOMM_H
#define SIMCOMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SIM_COMM_MAX_RANKS 64

typedef struct sim_comm* sim_comm_t;

typedef enum {
    COLL_OK = 0,
    COLL_ERR_INVALID_ARG = 1,
    COLL_ERR_UNSUPPORTED = 2,
    COLL_ERR_CUDA = 3,
    COLL_ERR_TIMEOUT = 4,
    COLL_ERR_ABORTED = 5,
    COLL_ERR_OVERFLOW = 6,
    COLL_ERR_INTERNAL = 7
} coll_status_t;

typedef enum { COLL_INT32 = 0, COLL_FP32 = 1, COLL_BF16 = 2 } coll_dtype_t;

typedef enum { COLL_SUM = 0, COLL_MIN = 1, COLL_MAX = 2, COLL_AVG = 3 } coll_op_t;

/* DIRECT: one fused pass reads all p inputs and writes every owner's output.
 * RING:   the ring schedule of [Atlas] §2.2, chunk-pipelined as in [Atlas] §3.5.
 * RD:     recursive doubling ([Atlas] §2.3): log2 p exchange-and-reduce steps. AllReduce only,
 *         p a power of two (else COLL_ERR_UNSUPPORTED).
 * HD:     recursive halving-doubling ([Atlas] §2.3): a halving reduce-scatter then a doubling
 *         all-gather, 2 log2 p steps. AllReduce only, p a power of two.
 * TREE:   reduce up a binary tree to its root, then broadcast down ([Primer] "Tree AllReduce 为什么
 *         更适合延迟敏感区间"): heap numbering, position m has children 2m+1 and 2m+2, rank m at
 *         position m; a position folds (own ⊕ left) ⊕ right in fp32; chunk-pipelined. AllReduce only.
 * DBTREE: double binary tree ([Atlas] §2.4): elements [0, ceil(n/2)) on the tree above, the rest on
 *         its mirror (rank p-1-m at position m). AllReduce only.
 * RING_LL: the ring schedule on the low-latency protocol of [Atlas] §3.4 (every 4 data bytes travel
 *         with a 4-byte flag in one 8-byte store; no separate flags or fences): same schedule and
 *         rounding as RING, so the same result bit for bit. AllReduce, ReduceScatter and AllGather;
 *         small messages: the communicator keeps p * (2p-3) (AllReduce) or p * (p-2) (the others)
 *         * ceil(n/p) * 8 bytes of receive slots, at most 256 MiB (else COLL_ERR_UNSUPPORTED).
 * RD_LL:  recursive doubling (as RD) on the LL protocol: same arithmetic as RD, so the same bits.
 *         AllReduce only, p a power of two, small messages: each rank's vector is held in registers
 *         of one resident grid (at most 8 elements per thread, about 1.2M / p elements on a B200)
 *         and p * log2(p) * n * 8 bytes of receive slots stay within 256 MiB (else
 *         COLL_ERR_UNSUPPORTED).
 * TREE_LL: the single binary tree (as TREE: same fold, so the same bits) on the LL protocol, any p;
 *         AllReduce only, small messages: p * 3 * n * 8 bytes of receive slots within 256 MiB.
 * DBTREE_LL: the double binary tree (as DBTREE: same split and fold, so the same bits) on the LL
 *         protocol, any p; AllReduce only, the same slot limit as TREE_LL. */
typedef enum {
    COLL_ALGO_DIRECT = 0, COLL_ALGO_RING = 1, COLL_ALGO_RD = 2, COLL_ALGO_HD = 3, COLL_ALGO_TREE = 4, COLL_ALGO_DBTREE = 5,
    COLL_ALGO_RING_LL = 6, COLL_ALGO_RD_LL = 7, COLL_ALGO_TREE_LL = 8, COLL_ALGO_DBTREE_LL = 9
} coll_algo_t;

typedef struct {
    const void* const* send; /* host array [p] of device pointers (inputs) */
    void* const* recv;       /* host array [p] of device pointers (outputs) */
} coll_bufs_t;

/* A cudaStream_t passed as an opaque pointer; NULL means the legacy default stream. */
typedef void* coll_stream_t;

/* ---- communicator lifecycle ([Primer] "Communicator 定义了“谁必须一起出现”") ----------------- */

/* Create a communicator of p ranks (1 <= p <= SIM_COMM_MAX_RANKS) on the current CUDA device.
 * Allocates its scratch (status words, ring flags; ring partial buffers grow on first use).
 * Returns NULL on failure; sim_comm_last_error() then says why. */
sim_comm_t sim_comm_create(int p);

/* A rank view: the handle that the process running rank `rank` of a p-rank communicator holds when
 * every rank is its own process (one per GPU, or several on one GPU), after [Atlas] §3.1-§3.3 (a
 * communicator's ranks exchange buffer handles once, then the P2P transport reads peers' buffers
 * directly). bufs.send[q] is then rank q's input as this process maps it (its own buffer for q =
 * rank, a mapping from sim_ipc_open of rank q's buffer otherwise) and bufs.recv[rank] this rank's
 * output; the other recv entries are ignored (may be NULL). A call computes this rank's output only,
 * reading the inputs it needs where they lie, with the direct path's kernels, fold order and
 * rounding, so the output equals the whole communicator's direct-path output for this rank bit for
 * bit. Supported: AllReduce, Reduce, Broadcast, ReduceScatter, AllGather, All-to-All, All-to-Allv
 * (counts_dev: this process's device copy of the whole count matrix, identical on every rank;
 * send_cap and recv_cap: every rank's capacities; only this rank's blocks are copied), Scatter,
 * Gather, COLL_ALGO_DIRECT only (the other schedules wait on other ranks inside their kernels:
 * COLL_ERR_UNSUPPORTED), and the MoE dispatch (fused kernel only) and combine (see there).
 * Reduce and Gather enqueue nothing
 * on a non-root rank. No output may overlap any rank's input (a peer may still be reading it), except
 * the root's own in-place Broadcast and Scatter forms. The ranks' calls are not synchronised by the
 * library: before a call every rank's inputs must be complete, and no rank may modify its input until
 * every rank's call that reads it has completed (e.g. every rank synchronises its stream and meets a
 * host barrier before and after each call). NULL on failure (p in [1, 64], rank in [0, p)). */
sim_comm_t sim_comm_create_rank(int p, int rank);

/* The rank of a rank view, -1 for a whole communicator, -2 for NULL. */
int sim_comm_rank(sim_comm_t comm);

/* Device memory another process can map (cudaIpcGetMemHandle / cudaIpcOpenMemHandle): the buffers
 * of a rank view's collectives. The handle is an opaque 64-byte value to send to the other ranks'
 * processes (by any host channel). */
typedef struct { unsigned char reserved[64]; } sim_ipc_handle_t;

/* Allocates `bytes` (> 0, at most 2^48) of device memory on the current device and its handle.
 * Free with sim_ipc_free in the same process, after every other process has closed its mapping. */
coll_status_t sim_ipc_alloc(size_t bytes, void** dev_ptr, sim_ipc_handle_t* handle);
coll_status_t sim_ipc_free(void* dev_ptr);

/* Maps another process's buffer into this one (*peer_ptr: its base as seen here; peer access between
 * GPUs is enabled on first use). A handle cannot be opened in the process that allocated it. Close
 * with sim_ipc_close before the owner frees the buffer. */
coll_status_t sim_ipc_open(const sim_ipc_handle_t* handle, void** peer_ptr);
coll_status_t sim_ipc_close(void* peer_ptr);

/* Free the communicator and its scratch. Synchronises the device first. NULL is accepted. */
coll_status_t sim_comm_destroy(sim_comm_t comm);

/* Number of ranks, or -1 for a NULL handle. */
int sim_comm_size(sim_comm_t comm);

/* Message of the last failed call on this thread (a static string owned by the library). */
const char* sim_comm_last_error(void);

/* Name of a status code (a static string). */
const char* coll_status_string(coll_status_t status);

/* Options (each also read from the environment at create time as SIMCOMM_<KEY upper-case>, e.g.
 * SIMCOMM_CHUNK_BYTES; a value the option rejects leaves the default):
 *   "chunk_bytes"  ring pipelining chunk in bytes of the reduce-scatter wire type (default 1 MiB,
 *                  a multiple of 256, [Atlas] §3.5)
 *   "ring_ctas"    CTAs of the ring executor (0 = as many as fit on the GPU; default 0)
 *   "ring_task_bytes"  bytes of the wire type one ring or tree task moves (a chunk is cut into tasks
 *                  of this size): 0 = by message size, 256 KiB from 64 MiB of wire bytes per rank
 *                  up, else 128 KiB (default); or a multiple of 256 in [4 KiB, 64 MiB]
 *   "timeout_ns"   longest device-side wait (a ring, tree or butterfly step for its predecessor, an
 *                  LL word, a bulk copy) before the call gives up with COLL_ERR_TIMEOUT (default 2e9)
 *   "fault_skip_rank"  debugging: this rank is silenced (the ring and tree executors never signal
 *                  its chunks, the butterfly executor never counts its tasks, the LL kernels never
 *                  send its words, and the fused MoE dispatch's CTA of this index never arrives at
 *                  its first grid barrier), so the waits on it time out (-1 = off, the default).
 *                  Host-side fault injection only.
 *   "copy_variant" copy path of the direct Broadcast/AllGather/All-to-All(v)/Scatter/Gather: -1 = the
 *                  default (Broadcast and AllGather: 9, the equal All-to-All: 11, where the buffers
 *                  allow it; the others: 6, 2 stages x 32 KiB, 3 CTAs per SM); 0..7 = a bulk-copy
 *                  pipeline shape (stages x tile bytes, CTAs per SM); 8 = the 16-byte load/store path
 *                  (All-to-All(v) only); 9..15 = the lean copy of Broadcast, AllGather and the equal
 *                  All-to-All (32 KiB tiles; 16-byte aligned buffers and whole 16-byte blocks, else 6):
 *                  9, 10 = 4 stages, 1 or 2 CTAs per SM; 11..14 = with lagged stage reuse, 4 stages
 *                  and 1 CTA per SM, 3 and 2, 6 and 1, 2 and 3; 15 = 6 stages, 1 CTA per SM;
 *                  16..18 = the equal All-to-All in one pass of 32-byte loads and stores, a CTA per
 *                  32, 64 or 16 KiB tile (32-byte aligned buffers and whole 32-byte blocks, else 6).
 *                  The bulk paths take their tiles in order from a shared counter; the one-pass
 *                  grid is handed out in order by the hardware.
 *   "copy_order"   tile order of the direct copy paths: -1 = the default per collective,
 *                  1 = interleaved over all blocks, 0 = block after block
 *   "direct_pack"  access width of the fused reduction: 0 = widest the alignment allows
 *                  (32 bytes), 16 = at most 16 bytes
 *   "direct_ctas_per_sm"  CTAs per SM of the fused reduction (default 16); 0 = one pass, a CTA per
 *                  iteration's worth of positions
 *   "l2_hint"      1 = evict-first L2 policy on the streaming loads and stores of the direct
 *                  paths (data read or written once), 2 = on the stores of the bulk-copy paths
 *                  only, 0 = none, -1 = per path (default; measured fastest): evict-first stores
 *                  where the lean fan-out of Broadcast or AllGather runs, none elsewhere
 *   "moe_fused"    coll_moe_dispatch as one cooperative kernel (counting, prefix sums and the copy
 *                  with grid barriers between them; 1, the default, where the device supports
 *                  cooperative launches) or as three kernels (0)
 *   "moe_tma"      copy kernel of the three-kernel coll_moe_dispatch: 0 = 32/16-byte loads and stores
 *                  (default, measured faster), 1 = bulk copies through shared memory (rows of whole
 *                  16-byte units at 16-byte aligned bases; otherwise the load/store kernel runs)
 *   "trace"        1 = keep a record of every call (sim_comm_trace_read), 0 = off (default).
 *                  Every entry point also opens an NVTX range named after its collective, whatever
 *                  this option says (a no-op unless a profiler collects NVTX).
 * Returns COLL_ERR_INVALID_ARG for an unknown key or a value out of range. */
coll_status_t sim_comm_set_option(sim_comm_t comm, const char* key, long long value);
coll_status_t sim_comm_get_option(sim_comm_t comm, const char* key, long long* value);

/* Non-blocking: *out receives COLL_OK or the first asynchronous error any kernel of this
 * communicator reported (polls a host-mapped word the kernels write; [Primer] section on failure
 * semantics: query the asynchronous error, abort, rebuild). */
coll_status_t sim_comm_get_async_error(sim_comm_t comm, coll_status_t* out);

/* Ask running and future ring steps to stop: a waiting step gives up with COLL_ERR_ABORTED.
 * Later calls return COLL_ERR_ABORTED until sim_comm_reset. Non-blocking. */
coll_status_t sim_comm_abort(sim_comm_t comm);

/* Wait for the device, clear the error state, the abort flag and the ring flags, so the
 * communicator can be used again. */
coll_status_t sim_comm_reset(sim_comm_t comm);

/* Kernels this communicator has launched so far (for launch accounting). */
coll_status_t sim_comm_launch_count(sim_comm_t comm, unsigned long long* out);

/* Per-call trace: the per-communicator record the [Primer] section "性能诊断第一步" asks for
 * (collective, count, dtype, group size, duration, algorithm), so that duration percentiles per
 * message size can be drawn from it. While option "trace" is 1 every entry-point call of this
 * communicator is recorded, with a CUDA event recorded on the caller's stream just before the
 * call's first kernel and one just after its last. */
typedef struct {
    unsigned long long seq;   /* number of the call among the traced calls of this communicator */
    const char* coll;         /* "allreduce", "reduce", ..., "moe_combine" (a static string) */
    int p;                    /* ranks */
    int dtype;                /* coll_dtype_t */
    int op;                   /* coll_op_t, or -1 where the call takes none */
    int root;                 /* root rank, or -1 where the call takes none */
    int algo;                 /* coll_algo_t, or -1 for the MoE calls */
    int status;               /* coll_status_t the call returned (asynchronous errors are not here) */
    unsigned long long n;     /* element count as passed; tokens for the MoE calls; 0 for All-to-Allv,
                                 whose counts stay on the device */
    unsigned int launches;    /* kernels the call enqueued */
    float device_ms;          /* time between the two events; -1 when the call launched nothing or its
                                 stream was being captured into a graph */
} sim_comm_trace_record_t;

/* Copies up to cap of the oldest records not read yet into out, in call order, and their number
 * into *count. Blocks until those calls' events have completed, so read off the hot path. The
 * communicator keeps the last 4096 traced calls; older unread records are lost (a gap in seq).
 * COLL_ERR_INVALID_ARG for a NULL comm or count, a negative cap, or a NULL out with cap > 0. */
coll_status_t sim_comm_trace_read(sim_comm_t comm, sim_comm_trace_record_t* out, int cap, int* count);

/* ---- collectives ------------------------------------------------------------------------------ */

/* AllReduce ([Atlas] §1.4; [Primer] "AllReduce：Partial 变成 Replicated"):
 * recv[r][i] = ⊕_q send[q][i] for every rank r, i < n. Identical results on every rank. */
coll_status_t coll_allreduce(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype,
                             coll_op_t op, coll_algo_t algo, coll_stream_t stream);

/* Reduce ([Atlas] §1.3, worked figure): recv[root][i] = ⊕_q send[q][i]. Only recv[root] is
 * written; the other recv pointers are ignored and may be NULL. */
coll_status_t coll_reduce(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype,
                          coll_op_t op, int root, coll_algo_t algo, coll_stream_t stream);

/* Broadcast ([Atlas] §1.1): recv[r][i] = send[root][i] for every rank r, the root included.
 * Only send[root] is read; the other send pointers are ignored and may be NULL. */
coll_status_t coll_broadcast(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype,
                             int root, coll_algo_t algo, coll_stream_t stream);

/* ReduceScatter ([Atlas] §1.5): with m = n/p, recv[r][k] = ⊕_q send[q][r·m + k], k < m.
 * send buffers hold n elements, recv buffers m. n must be divisible by p. */
coll_status_t coll_reduce_scatter(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype,
                                  coll_op_t op, coll_algo_t algo, coll_stream_t stream);

/* AllGather ([Atlas] §1.2): with m = n/p, recv[r][q·m + k] = send[q][k], k < m (shards
 * concatenated in rank order). send buffers hold m elements, recv buffers n. n divisible by p. */
coll_status_t coll_allgather(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype,
                             coll_algo_t algo, coll_stream_t stream);

/* All-to-All, equal split ([Atlas] §1.6): with m = n/p, recv[j][i·m + k] = send[i][j·m + k]
 * (the [src][dst] block matrix transposed). Both buffers hold n elements. n divisible by p. */
coll_status_t coll_alltoall(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype,
                            coll_algo_t algo, coll_stream_t stream);

/* Scatter ([Eight] "3.3 Scatter"; [Atlas] §0: the single-root form): with m = n/p,
 * recv[r][k] = send[root][r·m + k]. Only send[root] (n elements) is read; recv buffers hold m.
 * In place: recv[root] == send[root] + root·m. Direct path only (COLL_ALGO_RING:
 * COLL_ERR_UNSUPPORTED). */
coll_status_t coll_scatter(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype, int root,
                           coll_algo_t algo, coll_stream_t stream);

/* Gather ([Eight] "4.3 Gather"; [Atlas] §0): with m = n/p, recv[root][r·m + k] = send[r][k]. Only
 * recv[root] (n elements) is written; send buffers hold m. In place: send[root] == recv[root] +
 * root·m. Direct path only. */
coll_status_t coll_gather(sim_comm_t comm, coll_bufs_t bufs, size_t n, coll_dtype_t dtype, int root,
                          coll_algo_t algo, coll_stream_t stream);

/* All-to-Allv, uneven split ([Primer] "Ragged All-to-All：MoE 的真实输入通常不等长"):
 *   counts_dev   DEVICE int64 [p][p] row-major, c[i][j] = elements source i sends to destination j
 *                (the one matrix both sides read, so sends and receives always agree).
 *   send_cap     HOST int64 [p]: elements send[i] holds.   recv_cap  HOST int64 [p]: recv[j] holds.
 *   recv_counts_dev  DEVICE int64 [p] output Σ_i c[i][j], or NULL.
 * Source i packs its blocks in destination order, destination j stores them in source order:
 *   sdispl_i[j] = Σ_{j'<j} c[i][j'],  rdispl_j[i] = Σ_{i'<i} c[i'][j],
 *   recv[j][rdispl_j[i] + k] = send[i][sdispl_i[j] + k],  k < c[i][j].
 * The device checks every row sum against send_cap and every column sum against recv_cap; if any
 * count is negative or a sum exceeds its capacity, nothing is copied and the call reports
 * COLL_ERR_OVERFLOW asynchronously. counts_dev must stay unchanged until the call completes. */
coll_status_t coll_alltoallv(sim_comm_t comm, coll_bufs_t bufs, const long long* counts_dev,
                             const long long* send_cap, const long long* recv_cap, coll_dtype_t dtype,
                             coll_algo_t algo, coll_stream_t stream, long long* recv_counts_dev);

/* ---- MoE dispatch and combine ---------------------------------------------------------------- */

/* The steps on either side of the All-to-Allv in an expert-parallel MoE layer ([Primer] "Ragged
 * All-to-All：MoE 的真实输入通常不等长": router output -> count per destination -> exchange
 * counts -> prefix-sum offsets -> pack/permute -> variable-split exchange -> experts -> reverse
 * exchange -> unpermute/combine; [Primer] "Expert Parallel": one row travels per expert
 * assignment, and the combine weights the returned rows and adds the residual). Rules (our
 * reading): E experts, E a multiple of p, expert e lives on rank e / (E/p); every rank routes the
 * same number of tokens T, each to k experts (router output idx[t][s], t < T, s < k); rows hold H
 * elements, row-major, contiguous.
 *
 * Dispatch: counting, prefix sums, packing and the exchange in one call. Rank i's assignments are
 * packed by expert id, ties in token order then slot order; rank j receives [rows from rank 0 |
 * rows from rank 1 | ...], i.e. the All-to-Allv layout, every source block grouped by expert:
 *   x            HOST array of p DEVICE pointers, x[i] = [T][H] token rows of rank i.
 *   topk_idx     HOST array of p DEVICE pointers, [T][k] int32 expert ids in [0, E).
 *   recv         HOST array of p DEVICE pointers, [recv_cap_rows][H]; rows past the received
 *                count are left untouched.
 *   route_pos    HOST array of p DEVICE pointers [T][k] int32, or NULL: the row of recv[e/(E/p)]
 *                that received assignment (t, s), the routing map the combine needs.
 *   expert_counts_dev  DEVICE int64 [p][E] or NULL: assignments from rank i to expert e (expert e's
 *                rows from rank i follow those of the owner's lower experts inside rank i's block).
 *   recv_counts_dev    DEVICE int64 [p] or NULL: rows rank j received.
 * Any dtype (rows are copied bit for bit). Synchronous errors: k not in [1, 32], E not a multiple
 * of p in [p, 4096], H = 0, T*k or recv_cap_rows beyond int32, null or misaligned pointers,
 * overlapping outputs or an output overlapping an input. Asynchronous errors: an expert id outside
 * [0, E) -> COLL_ERR_INVALID_ARG, a rank that would receive more than recv_cap_rows rows ->
 * COLL_ERR_OVERFLOW; in both cases no row is copied. The scratch for counting is owned by the
 * communicator. T = 0 only zeroes the count outputs.
 * On a rank view (sim_comm_create_rank) x and topk_idx hold every rank's buffers as this process
 * maps them, recv and route_pos only this rank's entry (the others are ignored), and the count
 * outputs are this process's own arrays; each rank counts every rank's assignments and copies the
 * rows destined to itself, so its outputs equal the whole communicator's for this rank bit for bit.
 * Needs option moe_fused = 1 (else COLL_ERR_UNSUPPORTED). */
coll_status_t coll_moe_dispatch(sim_comm_t comm, const void* const* x, const int32_t* const* topk_idx, size_t tokens,
                                int k, size_t hidden, int experts, coll_dtype_t dtype, void* const* recv,
                                size_t recv_cap_rows, int32_t* const* route_pos, long long* expert_counts_dev,
                                long long* recv_counts_dev, coll_stream_t stream);

/* Combine: reverse exchange, unpermute and weighted sum in one call:
 *   out[i][t] = residual[i][t] + Σ_{s<k} w[i][t][s] * y[e/(E/p)][route_pos[i][t][s]],  e = idx[i][t][s]
 * accumulated in fp32 in slot order (the residual first; without a residual the sum starts at the
 * slot-0 product), every product and sum rounded to fp32, then rounded once to the row type.
 *   y            HOST array of p DEVICE pointers, [y_rows][H]: expert outputs in the dispatch's
 *                receive layout (e.g. recv after the experts ran in place).
 *   topk_idx, route_pos  as given to and returned by coll_moe_dispatch.
 *   topk_weight  HOST array of p DEVICE pointers, [T][k] fp32 gate weights.
 *   residual     HOST array of p DEVICE pointers [T][H], or NULL (no residual term); residual[i]
 *                may equal out[i] (in place).
 *   out          HOST array of p DEVICE pointers [T][H].
 * dtype fp32 or bf16 (int32 -> COLL_ERR_UNSUPPORTED). An expert id outside [0, E) or a route_pos
 * outside [0, y_rows) is reported asynchronously as COLL_ERR_INVALID_ARG (that token is skipped).
 * On a rank view y holds every rank's expert outputs as this process maps them, and topk_idx,
 * route_pos, topk_weight, residual and out only this rank's entry: the call combines this rank's
 * tokens, reading the rows they were routed to where they lie. */
coll_status_t coll_moe_combine(sim_comm_t comm, const void* const* y, size_t y_rows, const int32_t* const* topk_idx,
                               const int32_t* const* route_pos, const float* const* topk_weight,
                               const void* const* residual, size_t tokens, int k, size_t hidden, int experts,
                               coll_dtype_t dtype, void* const* out, coll_stream_t stream);

/* ---- diagnostics ------------------------------------------------------------------------------ */

/* HBM access-pattern probe (not a collective; the pages have no counterpart): streams `bytes` through
 * HBM with one access pattern of the library's kernels, so that a kernel's throughput can be read
 * against the ceiling of its own pattern on this device.
 *   kind  0 = load only (32-byte loads of src; their XOR is compared with a constant, and only in
 *             the practically never taken equal case is one word written to dst[0..3], if dst is
 *             not NULL),
 *         1 = store only (32-byte stores of a fixed pattern to dst),
 *         2 = copy (32-byte loads of src, stored to dst),
 *         3 = bulk store only (cp.async.bulk stores of one 16 KiB shared-memory tile to dst, one warp
 *             per CTA: the fan-out side of Broadcast and AllGather),
 *         4 = bulk fan-out 1:8 (every 32 KiB tile of src loaded once into shared memory and stored
 *             to dst + f·bytes for f = 0..7, tiles claimed in order: the whole Broadcast / AllGather
 *             pattern of 8 ranks; dst holds 8·bytes). Not re-entrant: its tile counter is a device
 *             variable of the library, so two kind-4 probes must not overlap on the GPU.
 *   dst, src  DEVICE pointers, 256-byte aligned, non-overlapping; src is unused by kinds 1 and 3, dst
 *             by kind 0 (either may then be NULL).
 *   bytes     a multiple of 16 KiB (kind 4: of 32 KiB, at most 2^40; 0: nothing is enqueued).
 *   ctas_per_sm  CTAs per SM of a persistent grid-stride grid, in [1, 32]; 0 = one pass (kinds 0-3:
 *             a CTA per 32 KiB of the loop or per 16 KiB tile, dispatched in address order as SMs free
 *             up; kind 4: one CTA per SM).
 * Enqueues one kernel on the stream. COLL_ERR_INVALID_ARG for a bad kind, size, pointer or overlap. */
coll_status_t sim_hbm_probe(int kind, void* dst, const void* src, size_t bytes, int ctas_per_sm,
                            coll_stream_t stream);

/* ---- no-allocation variant ------------------------------------------------------------------ */

/* Ring AllReduce that allocates nothing. (The pages have no counterpart: this is a library
 * facility, not part of the collective's definition.)
 *
 * For callers that cannot call cudaMalloc: code inside a memory pool or allocator (which must not
 * re-enter the allocator it implements), a process that must not grow its device footprint after
 * start-up (its memory is budgeted up front, and cudaMalloc may also synchronise the device), or code
 * that runs where a framework forbids allocation. It computes exactly what
 * coll_allreduce(..., COLL_ALGO_RING, ...) computes on a communicator of p ranks with default options
 * (same kernel, same schedule and tiling, same rounding), but needs no communicator: its scratch
 * (control words, chunk flags, one fp32/int32 partial buffer per rank) is a fixed 32 MiB device array
 * inside the library, held on every GPU that loads the library until the process exits.
 *   p, bufs, n, dtype, op  as for coll_allreduce (2 <= p <= 64).
 *   async_status_dev  DEVICE int the caller owns, or NULL: receives COLL_OK or the asynchronous
 *                     error of this call (COLL_ERR_TIMEOUT if a ring step waited longer than the
 *                     timeout), in stream order.
 * Two settings are read from the environment at every call, as a communicator reads its options at
 * create time: SIMCOMM_TIMEOUT_NS, the longest wait of a ring step (default 2e9, at least 1000), and
 * SIMCOMM_FAULT_SKIP_RANK, host-side fault injection (that rank never signals, so its successor
 * times out; -1 = off, the default). A value out of range leaves the default.
 * Limits and errors: the scratch must hold p * round_up(4n, 256) bytes of partials plus the flags
 * (about p * n * 4 < 32 MiB, e.g. n up to ~1M elements at p = 8); larger calls return
 * COLL_ERR_INVALID_ARG with the sizes in sim_comm_last_error(). Other argument errors as for
 * coll_allreduce. The first call on a device looks up the scratch's device address on that device
 * and keeps it for the life of the process; after
 * cudaDeviceReset or any other teardown of the device's primary context that address is stale, so
 * do not call this entry point again in that process. Every call shares the scratch and clears what
 * must start at zero on its own stream; calls that overlap on the GPU race on it and must be
 * ordered by the caller. */
coll_status_t coll_allreduce_ring_noalloc(int p, coll_bufs_t bufs, size_t n, coll_dtype_t dtype, coll_op_t op,
                                          int* async_status_dev, coll_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SIMCOMM_H */
