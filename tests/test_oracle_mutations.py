"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pins catch each.

Every mutant is compiled from a textual edit of oracle.cpp into a temporary directory; the pin
suite then runs against it in a subprocess and must fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.cpp")

MUTANTS = {
    "drop_last_rank_exact": ("for (int k = 1; k < p; ++k) s += load_as_double", "for (int k = 1; k < p - 1; ++k) s += load_as_double"),
    "min_max_swapped": ("if (op == OP_MIN) return (b < a) ? b : a;", "if (op == OP_MIN) return (b > a) ? b : a;"),
    "allgather_wrong_block": ("copy_element(in[q], k, out[r], size_t(q) * m + k, dtype)", "copy_element(in[q], k, out[r], size_t(r) * m + k, dtype)"),
    "alltoall_untransposed": ("copy_element(in[i], size_t(j) * m + k, out[j], size_t(i) * m + k, dtype)", "copy_element(in[i], size_t(i) * m + k, out[j], size_t(j) * m + k, dtype)"),
    "reduce_scatter_wrong_owner": ("reduce_element(p, in, order, size_t(r) * m + k, dtype, op, acc, out[r], k)", "reduce_element(p, in, order, size_t((r + 1) % p) * m + k, dtype, op, acc, out[r], k)"),
    "ring_wrong_chunk": ("int c = mod(r - s, p);", "int c = mod(r - s - 1, p);"),
    "alltoallv_rdispl_transposed": ("rdispl += counts[ii * p + j]", "rdispl += counts[j * p + ii]"),
    "bf16_ties_away": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;", "if (lower >= 0x8000u) upper += 1;"),
    "avg_not_scaled": ("if (op == OP_AVG) s = s / double(p);", ""),
    "ring_broadcast_wrong_hop": ("int src = mod(root + h - 1, p), dst = mod(root + h, p);", "int src = mod(root + h - 1, p), dst = mod(root + h + 1, p);"),
    "double_bf16_wrong_quantum": ("int q = e - 8;", "int q = e - 9;"),
    "ring_avg_scale_missing": ("if (op == OP_AVG) { volatile float scale = 1.0f / float(p); v = v * scale; }\n        store_float(out, dtype, oi, v);\n    }\n};", "store_float(out, dtype, oi, v);\n    }\n};"),
    "rd_wrong_partner": ("const int lo = std::min(r, r ^ d), hi = std::max(r, r ^ d);", "const int lo = std::min(r, (r + d) % p), hi = std::max(r, (r + d) % p);"),
    "hd_ascending_halving": ("for (int d = p / 2; d >= 1; d >>= 1) {", "for (int d = 1; d < p; d <<= 1) {"),
    "hd_keeps_wrong_half": ("const int kb = (r & d) ? group + d : group;", "const int kb = (r & d) ? group : group + d;"),
    "scatter_wrong_block": ("copy_element(in_root, size_t(r) * m + k, out[r], k, dtype);", "copy_element(in_root, size_t((r + 1) % p) * m + k, out[r], k, dtype);"),
    "gather_wrong_block": ("copy_element(in[r], k, out_root, size_t(r) * m + k, dtype);", "copy_element(in[r], k, out_root, size_t(p - 1 - r) * m + k, dtype);"),
    "moe_ties_reversed": ("std::stable_sort(ord.begin(), ord.end(), [ids](int64_t x, int64_t y) { return ids[x] < ids[y]; });", "std::sort(ord.begin(), ord.end(), [ids](int64_t x, int64_t y) { return ids[x] < ids[y] || (ids[x] == ids[y] && x > y); });"),
    "moe_owner_modulo": ("R->c[size_t(i) * p + e / R->E_loc] += 1;", "R->c[size_t(i) * p + e % p] += 1;"),
    "moe_pos_no_source_offset": ("for (int ii = 0; ii < i; ++ii) rdispl += R.c[size_t(ii) * p + j];", ""),
    "moe_pack_wrong_token": ("const size_t t = size_t(R.order[i][q]) / size_t(k);", "const size_t t = size_t(R.order[i][q]) % T;"),
    "moe_combine_weight_slot_swapped": ("sum += double(w[i][t * k + s]) *", "sum += double(w[i][t * k + (k - 1 - s)]) *"),
    "moe_combine_drops_residual": ("double sum = residual ? load_as_double(residual[i], dtype, t * H + h) : 0.0;", "double sum = 0.0;"),
    "moe_reverse_untransposed": ("ct[size_t(j) * p + i] = R.c[size_t(i) * p + j] * int64_t(H);", "ct[size_t(i) * p + j] = R.c[size_t(i) * p + j] * int64_t(H);"),
    "tree_children_swapped": ("for (int c = 2 * m + 1; c <= 2 * m + 2 && c < p; ++c) {", "for (int c = std::min(2 * m + 2, p - 1); c >= 2 * m + 1; --c) {"),
    "tree_b_not_mirrored": ("const int r = mirror ? p - 1 - m : m;", "const int r = m;"),
    "tree_split_floor": ("const size_t half = double_tree ? (n + 1) / 2 : n;", "const size_t half = double_tree ? n / 2 : n;"),
    "int_sum_saturates": ("if (op == OP_SUM) i[k] = int32_t(uint32_t(received_i) + uint32_t(o));", "if (op == OP_SUM) i[k] = int32_t(std::max<int64_t>(INT32_MIN, std::min<int64_t>(INT32_MAX, int64_t(received_i) + o)));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {name}"
    mutant = src.replace(old, new)
    if name == "int_sum_saturates":
        mutant = "#include <algorithm>\n#include <climits>\n" + mutant
    cpp = tmp_path / "oracle_mutant.cpp"
    cpp.write_text(mutant)
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-o", str(lib), str(cpp)],
                   check=True)
    env = dict(os.environ, ORACLE_LIB=str(lib))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                          os.path.join(ROOT, "tests", "test_oracle_rd_hd.py"),
                          os.path.join(ROOT, "tests", "test_oracle_rooted.py"),
                          os.path.join(ROOT, "tests", "test_oracle_moe.py"),
                          os.path.join(ROOT, "tests", "test_oracle_tree.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"mutant {name} survived the pins:\n{res.stdout[-2000:]}"
