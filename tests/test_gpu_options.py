"""Communicator options (sim_comm_set_option / sim_comm_get_option, include/simcomm.h): every key
takes the values its documentation gives and refuses the rest with COLL_ERR_INVALID_ARG, a refused
value leaves the option as it was, and an unknown key is refused. No collective runs."""
import pytest

from collective_communication_primitives_b200 import simcomm as SC

pytestmark = pytest.mark.gpu

P = 4
OPTIONS = {
    # key: (accepted, refused)
    "chunk_bytes": ([256, 1 << 20, 1 << 30], [0, 255, 257, (1 << 30) + 256]),
    "ring_ctas": ([0, 1, 65535], [-1, 65536]),
    "timeout_ns": ([1000, 2_000_000_000], [999, 0, -5]),
    "fault_skip_rank": ([-1, 0, P - 1], [-2, P]),
    "copy_variant": ([-1, 0, 8, 9, 18], [-2, 19]),
    "copy_order": ([-1, 0, 1], [-2, 2]),
    "l2_hint": ([-1, 0, 1, 2], [-2, 3]),
    "direct_pack": ([0, 16, 32], [8, 64, -1]),
    "direct_ctas_per_sm": ([0, 16, 32], [-1, 33]),
    "ring_task_bytes": ([0, 4096, 64 << 20], [256, 4095, 4096 + 128, (64 << 20) + 256]),
    "moe_tma": ([0, 1], [-1, 2]),
    "moe_fused": ([0, 1], [-1, 2]),
    "trace": ([0, 1], [-1, 2]),
}


def test_every_option_takes_its_range_and_refuses_the_rest():
    with SC.SimComm(P) as c:
        for key, (good, bad) in OPTIONS.items():
            for v in good:
                c.set_option(key, v)
                assert c.get_option(key) == v, (key, v)
            for v in bad:
                with pytest.raises(SC.SimCommError) as e:
                    c.set_option(key, v)
                assert e.value.status == SC.INVALID_ARG, (key, v)
                assert c.get_option(key) == good[-1], (key, v)  # a refused value changes nothing
        with pytest.raises(SC.SimCommError) as e:
            c.set_option("no_such_option", 1)
        assert e.value.status == SC.INVALID_ARG
        with pytest.raises(SC.SimCommError) as e:
            c.get_option("no_such_option")
        assert e.value.status == SC.INVALID_ARG
