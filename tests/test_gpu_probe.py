"""The HBM access-pattern probe (sim_hbm_probe) moves exactly what it says: the copy reproduces its
source, the stores write their fixed pattern, the bulk fan-out writes 8 copies, the load-only probe
leaves its destination alone; bad sizes, alignments and overlaps are refused before any launch."""
import ctypes

import numpy as np
import pytest
import torch

from collective_communication_primitives_b200 import simcomm as SC

pytestmark = pytest.mark.gpu

NB = 1 << 20  # bytes: 64 tiles of 16 KiB, 32 of 32 KiB


def src_words():
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    return torch.randint(-2**31, 2**31 - 1, (NB // 4,), dtype=torch.int32, device="cuda", generator=g)


@pytest.mark.parametrize("cps", [0, 2])
def test_copy_store_load(cps):
    src = src_words()
    dst = torch.zeros(NB // 4, dtype=torch.int32, device="cuda")
    SC.hbm_probe("copy", dst, src, NB, cps)
    torch.cuda.synchronize()
    assert torch.equal(dst, src)
    SC.hbm_probe("store", dst, None, NB, cps)
    torch.cuda.synchronize()
    want = (np.uint32(0x3C003C00) + np.arange(8, dtype=np.uint32)).view(np.int32)
    assert np.array_equal(dst.view(-1, 8).cpu().numpy(), np.broadcast_to(want, (NB // 32, 8)))
    before = dst.clone()
    SC.hbm_probe("load", dst, src, NB, cps)
    torch.cuda.synchronize()
    assert torch.equal(dst, before)


@pytest.mark.parametrize("cps", [0, 4])
def test_bulk_store_pattern(cps):
    dst = torch.zeros(NB // 4, dtype=torch.int32, device="cuda")
    SC.hbm_probe("bulk_store", dst, None, NB, cps)
    torch.cuda.synchronize()
    w = np.arange(4096)
    tile = (16 * (w // 4) + (w % 4)).astype(np.int32)  # word w of a 16 KiB tile: its 16-byte unit's offset + w mod 4
    assert np.array_equal(dst.view(-1, 4096).cpu().numpy(), np.broadcast_to(tile, (NB // 16384, 4096)))


def test_bulk_fanout_writes_eight_copies():
    src = src_words()
    dst = torch.zeros(8 * NB // 4, dtype=torch.int32, device="cuda")
    SC.hbm_probe("bulk_fanout", dst, src, NB, 1)
    torch.cuda.synchronize()
    for f in range(8):
        assert torch.equal(dst[f * NB // 4:(f + 1) * NB // 4], src), f
    SC.hbm_probe("bulk_fanout", dst, src, NB, 2)  # its tile counter was reset by the previous call
    torch.cuda.synchronize()
    assert torch.equal(dst[-NB // 4:], src)


def test_bad_arguments_are_refused():
    L = SC.load_library()
    a = torch.zeros(NB // 4 + 64, dtype=torch.int32, device="cuda")
    b = torch.zeros(NB // 4, dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    vp = lambda t, off=0: ctypes.c_void_p(t.data_ptr() + off)
    assert L.sim_hbm_probe(2, vp(b), vp(a), NB - 16, 1, s) == SC.INVALID_ARG        # not whole 16 KiB tiles
    assert L.sim_hbm_probe(2, vp(b), vp(a, 16), NB, 1, s) == SC.INVALID_ARG         # not 256-byte aligned
    assert L.sim_hbm_probe(2, vp(a, 256), vp(a), NB, 1, s) == SC.INVALID_ARG        # overlapping
    assert L.sim_hbm_probe(4, vp(b), vp(a), NB - 16384, 1, s) == SC.INVALID_ARG     # fan-out: not whole 32 KiB tiles
    assert L.sim_hbm_probe(9, vp(b), vp(a), NB, 1, s) == SC.INVALID_ARG             # unknown kind
    assert L.sim_hbm_probe(2, vp(b), vp(a), NB, 33, s) == SC.INVALID_ARG            # ctas_per_sm out of range
    assert L.sim_hbm_probe(1, None, None, NB, 1, s) == SC.INVALID_ARG               # null destination
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(b)) == 0  # nothing ran
