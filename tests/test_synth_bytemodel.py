"""Host-side logic: the seeded input generators and the byte model."""
import numpy as np
import pytest

from collective_communication_primitives_b200 import bytemodel as B
from collective_communication_primitives_b200 import synth as S


def test_generators_are_deterministic_and_counter_based():
    a = S.normal("x", 10_000_000, 1e-3)
    b = S.normal("x", 10_000_000, 1e-3)
    np.testing.assert_array_equal(a, b)
    # any element can be drawn alone: a prefix equals the start of a longer draw
    np.testing.assert_array_equal(S.normal("x", 1000, 1e-3), a[:1000])
    assert not np.array_equal(S.normal("y", 1000, 1e-3), a[:1000])
    assert not np.array_equal(S.normal("x", 1000, 1e-3, seed=1), a[:1000])


def test_distributions():
    x = S.normal("n", 2_000_000, 0.02).astype(np.float64)
    assert abs(x.mean()) < 1e-4 and abs(x.std() - 0.02) < 1e-4
    i = S.ints("i", 1_000_000, -8, 8)
    assert i.min() == -8 and i.max() == 8 and abs(i.mean()) < 0.02
    u = S.uniform_pm1("u", 1_000_000)
    assert u.min() >= -1.0 and u.max() < 1.0 and abs(u.mean()) < 0.01
    assert np.all(np.ldexp(u.astype(np.float64), 23) == np.round(np.ldexp(u.astype(np.float64), 23)))


def test_bf16_encoding_rounds_to_nearest_even():
    import torch
    x = S.normal("b", 100_000, 1.0)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(S.normal("b", 100_000, 1.0, "bf16"), ref)


def test_moe_counts_shape_and_skew():
    c = S.moe_counts()
    rows = c // 4096
    assert c.shape == (8, 8) and np.all(c % 4096 == 0)
    assert np.all(rows.sum(axis=1) == 8192 * 2)          # top-2: two assignments per token
    assert rows.sum(axis=0).argmax() == 0                 # rank 0 holds the most popular experts
    assert np.all(rows.sum(axis=0)[:-1] >= rows.sum(axis=0)[1:])
    st = S.count_matrix_stats(rows)
    assert st["max_row"] == 16384 and st["max_col"] <= 8 * 16384
    np.testing.assert_array_equal(S.moe_counts(), c)


def test_byte_model_pins():
    # "8 primitives" blog §6.2: TP AllReduce of one H = 8192 fp16 activation row over N = 8 ranks
    # moves about 2 * 8192 * 2 * 0.875 bytes = 28,672 B per rank.
    assert B.ring_wire_bytes_per_rank("allreduce", 8, 8192 * 2) == 28672
    # the same section's MoE example: 1,024 tokens of H = 8192 fp16 per card, 63/64 of them routed
    # away (64 destinations): 1008 * 2 * 8192 bytes sent per card, about 16 MB, and eight cards'
    # worth, about 128 MB per layer
    per_card = B.ring_wire_bytes_per_rank("alltoall", 64, 1024 * 2 * 8192)
    assert per_card == 1008 * 2 * 8192 == 16_515_072
    assert 8 * per_card == 132_120_576
    # Atlas §2.5 bus-bandwidth factors
    assert B.busbw_factor("allreduce", 8) == pytest.approx(1.75)
    assert B.busbw_factor("reduce_scatter", 4) == pytest.approx(0.75)
    assert B.busbw_factor("allgather", 4) == pytest.approx(0.75)
    assert B.busbw_factor("alltoall", 64) == pytest.approx(63 / 64)
    assert B.busbw_factor("broadcast", 8) == 1.0 and B.busbw_factor("reduce", 8) == 1.0
    # direct path: AllReduce reads p·n and writes p·n
    assert B.direct_hbm_bytes("allreduce", 8, 1000, 4) == 64000
    assert B.direct_hbm_bytes("allreduce", 8, 1000, 2) == 32000
    assert B.direct_hbm_bytes("reduce_scatter", 8, 1000, 2) == 18000
    assert B.direct_hbm_bytes("allgather", 8, 1000, 2) == 18000
    assert B.direct_hbm_bytes("alltoallv", 8, 0, 2, moved_elems=10) == 40


def test_ring_byte_model_counts_hops():
    p, n, d = 8, 8000, 4
    seg = n // p
    # reduce-scatter phase: p segments, each through p-1 hops of (read, read, write) = 3 segs each
    assert B.ring_hbm_bytes("reduce_scatter", p, n, d) == p * (p - 1) * 3 * seg * d
    assert B.ring_hbm_bytes("allreduce", p, n, d) == p * (p - 1) * 3 * seg * d + p * (p - 1) * 2 * seg * d
    # bf16 with fp32 partials
    hb = B.ring_hbm_bytes("allreduce", p, n, 2, 4)
    assert hb == n * ((2 * 2 + 4) + (p - 3) * (2 * 4 + 2) + (4 + 2 * 2)) + (p - 1) * n * 2 * 2
