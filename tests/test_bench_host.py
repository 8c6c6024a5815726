"""Host-side checks of bench.py that need no GPU: the step's row list, the shared `config` of both
arms and the reference arm's JSON line (it times the oracle on the host)."""
import io
import json
import types
from contextlib import redirect_stdout

import bench


def test_step_rows_match_build_step():
    wl = types.SimpleNamespace(n=8 * 1024, p=bench.P, v_elems=1000, x32=None, x16=None, ar32=None, ar16=None,
                               red=None, out32=None, rs=None, shards=None, v_send=None, v_recv=None, counts=None)
    names = [o[0] for o in bench.build_step(object(), wl)]
    assert tuple(names) == bench.STEP_ROWS


def test_reference_arm_line_matches_this_arms_contract():
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=1, option=[])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_arm(args)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["config"] == bench.step_config(bench.N_BUCKET, 1, list(bench.STEP_ROWS), [])
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_moe_byte_models():
    from collective_communication_primitives_b200 import bytemodel as BM
    # 8 ranks x 8192 tokens, top-2, 4096-wide bf16 rows
    assert BM.moe_dispatch_bytes(8, 8192, 2, 4096, 2) == 8 * (8192 * 4096 * 2 + 16384 * 4096 * 2 + 8 * 16384)
    assert BM.moe_combine_bytes(8, 8192, 2, 4096, 2) == 8 * (16384 * 4096 * 2 + 2 * 8192 * 4096 * 2 + 12 * 16384)
    assert BM.moe_combine_bytes(1, 1, 1, 1, 4, residual=False) == 4 + 4 + 12


def test_oracle_slices_cover_the_bucket_and_threads_agree():
    """The all-cores CPU baseline cuts the step into contiguous ranges that tile every rank's bucket;
    each range is an independent step whose elementwise rows equal the full step's on that range."""
    import numpy as np

    import oracle as O
    n = bench.P * 64 * 10 + bench.P * 64 * 3  # 13 units: ragged against 4 threads
    inp = bench.oracle_inputs(n)
    parts = bench.oracle_slices(inp, 4)
    assert sum(q["n"] for q in parts) == n and all(q["n"] % (bench.P * 64) == 0 for q in parts)
    lo = 0
    full = O.allreduce(inp["x32"], "fp32", "avg", acc="rankfold")
    for q in parts:
        assert q["x32"][0].base is not None or q["x32"][0] is inp["x32"][0]  # views, no copies
        np.testing.assert_array_equal(q["x32"][3], inp["x32"][3][lo:lo + q["n"]])
        got = O.allreduce(q["x32"], "fp32", "avg", acc="rankfold")
        np.testing.assert_array_equal(got[0], full[0][lo:lo + q["n"]])
        assert int(q["counts"].sum(axis=1).max()) <= q["n"]
        lo += q["n"]
    secs, eff, used = bench.oracle_step_threads(inp, 4)
    assert used == len(parts) and secs > 0 and eff > 0
