"""Byte models of the collectives: the HBM bytes one call must move on a simulated communicator,
the logical wire bytes of the ring schedule, and bus-bandwidth factors.

Notation: p ranks, n = the per-rank full-buffer element count (the AllReduce in/out size, the
ReduceScatter input size, the AllGather output size, the All-to-All send size), d = bytes per
element.

Sources:
  [Atlas] "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives),
          §2.2 ring all-reduce cost, §2.5 bus bandwidth factor table.
  [Primer] "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All",
          section "先统一通信量的记号" (per-rank wire bytes exclude the self-copy).
"""

OPS = ("allreduce", "reduce", "broadcast", "reduce_scatter", "allgather", "alltoall", "alltoallv")


def direct_hbm_bytes(op, p, n, d_in, d_out=None, moved_elems=None):
    """Minimum HBM bytes of one call when all p ranks share one GPU's memory: every input element
    read once, every output element written once.

    alltoallv takes ``moved_elems`` = Σ_ij c_ij (the count matrix itself is negligible).
    Broadcast and AllGather are counted out of place (the root's / each shard's own copy included).
    """
    d_out = d_in if d_out is None else d_out
    if op == "allreduce":
        return p * n * d_in + p * n * d_out
    if op == "reduce":
        return p * n * d_in + n * d_out
    if op == "broadcast":
        return n * d_in + p * n * d_out
    if op == "reduce_scatter":
        return p * n * d_in + n * d_out
    if op == "allgather":
        return n * d_in + p * n * d_out
    if op == "alltoall":
        return p * n * d_in + p * n * d_out
    if op == "alltoallv":
        if moved_elems is None:
            raise ValueError("alltoallv needs moved_elems")
        return moved_elems * (d_in + d_out)
    raise ValueError(op)


def _chain_bytes(p, elems, d, a):
    """HBM bytes of p-1 reduce hops over ``elems`` elements: each hop reads the predecessor's
    partial and its own input and writes a partial; the first hop's partial is a raw input (d),
    the last hop writes the output (d); partials in between are a bytes each."""
    if p == 1:
        return 2 * elems * d                      # the own input copied to the output
    if p == 2:
        return elems * 3 * d
    return elems * ((2 * d + a) + (p - 3) * (2 * a + d) + (a + 2 * d))


def ring_hbm_bytes(op, p, n, d, acc_d=None, moved_elems=None):
    """HBM bytes the simulated ring schedule moves (reported, not a target).

    A reduce hop reads the predecessor's partial and its own input and writes its partial; partials
    are acc_d bytes (4 for bf16 data, else d). A copy hop reads d and writes d. In the reduce-scatter
    phase every one of the p segments goes through its own chain of p-1 hops; in the all-gather
    phase every rank receives p-1 segments. A self-copy (the own shard, the root's own output) is a
    read and a write.
    """
    a = d if acc_d is None else acc_d
    if op == "allreduce":
        return _chain_bytes(p, n, d, a) + (p - 1) * n * 2 * d
    if op == "reduce_scatter":
        return _chain_bytes(p, n, d, a)
    if op == "reduce":
        return _chain_bytes(p, n, d, a)
    if op == "broadcast":
        return 2 * n * d * p                      # root's own copy plus p-1 hops
    if op == "allgather":
        return 2 * n * d * p                      # own shard plus p-1 received shards, per rank
    if op in ("alltoall", "alltoallv"):
        return direct_hbm_bytes(op, p, n, d, d, moved_elems)
    raise ValueError(op)


def ring_wire_bytes_per_rank(op, p, n_bytes):
    """Logical bytes one rank sends in the ring schedule, self-copy excluded ([Atlas] §2.2 and
    §2.5): AllReduce 2(p-1)/p·B, ReduceScatter/AllGather/All-to-All (p-1)/p·B, Broadcast/Reduce B.
    B is the per-rank full buffer in bytes (the AllGather output, the ReduceScatter input)."""
    return busbw_factor(op, p) * n_bytes


def busbw_factor(op, p):
    """Bus-bandwidth correction factor of [Atlas] §2.5: busbw = algbw × factor."""
    if op == "allreduce":
        return 2.0 * (p - 1) / p
    if op in ("reduce_scatter", "allgather", "alltoall", "alltoallv"):
        return (p - 1) / p
    if op in ("broadcast", "reduce"):
        return 1.0
    raise ValueError(op)


def moe_dispatch_bytes(p, tokens, k, hidden, d):
    """Minimum HBM bytes of one MoE dispatch over p ranks: every token row read once, every
    assignment row (k per token) written once, the expert ids read and the routing map written
    (4 bytes per assignment each); the per-tile counting scratch is not counted."""
    a = tokens * k
    return p * (tokens * hidden * d + a * hidden * d + 2 * 4 * a)


def moe_combine_bytes(p, tokens, k, hidden, d, residual=True):
    """Minimum HBM bytes of one MoE combine over p ranks: every assignment's expert-output row read
    once, the residual read (when given) and the output written once per token, and the expert id,
    routing-map entry and gate weight read per assignment (4 bytes each)."""
    a = tokens * k
    return p * (a * hidden * d + (2 if residual else 1) * tokens * hidden * d + 3 * 4 * a)
