"""Each planted mistake in a copy of the oracle must fail at least one pin.

The copies are compiled from the oracle's C source with one text edit each
(a dropped term, a wrong sign, index or order, a transposed operand), on the
CPU.  This shows the pins in oracle_checks.py are strong enough to catch
plausible errors in every step of the oracle."""
import ctypes
import os
import subprocess
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import oracle_checks as oc  # noqa: E402

MUTANTS = {
    "sequential_router_sum": ("const int p = (int)(i % 32);", "const int p = 0;"),
    "unfused_router_fma": ("fmaf(xi, wr[e], v[e * 32 + p])", "xi * wr[e] + v[e * 32 + p]"),
    "neighbour_butterfly": ("for (int m = 16; m >= 1; m >>= 1)", "for (int m = 1; m <= 16; m <<= 1)"),
    "router_bias_sign": ("l = l + b_r[e];", "l = l - b_r[e];"),
    "tie_to_higher_id": ("l[e] > l[best]", "l[e] >= l[best]"),
    "softmax_sign": ("exp((double)l[idx[j]] - l0)", "exp(l0 - (double)l[idx[j]])"),
    "offsets_off_by_one": ("offsets[e + 1] = offsets[e] + counts[e];",
                           "offsets[e + 1] = offsets[e] + counts[e] + (e == 0);"),
    "scatter_stores_token": ("sorted_assign[p] = (int32_t)a;", "sorted_assign[p] = (int32_t)(a / k);"),
    "block_rows_not_clipped": ("? counts[e] - i * BT : BT", "? BT : BT"),
    # an expert's rows split evenly over its tiles (300 rows at BT 128: 100/100/100)
    "block_even_split": (
        "const int64_t rows = counts[e] - i * BT < BT ? counts[e] - i * BT : BT;\n"
        "            block_map[3 * nb + 0] = (int32_t)e;\n"
        "            block_map[3 * nb + 1] = (int32_t)(offsets[e] + i * BT);",
        "const int64_t per = (counts[e] + tiles - 1) / tiles;\n"
        "            const int64_t rows = i == tiles - 1 ? counts[e] - per * (tiles - 1) : per;\n"
        "            block_map[3 * nb + 0] = (int32_t)e;\n"
        "            block_map[3 * nb + 1] = (int32_t)(offsets[e] + i * per);"),
    # the ragged tile first (300 rows at BT 128: 44/128/128)
    "block_ragged_first": (
        "const int64_t rows = counts[e] - i * BT < BT ? counts[e] - i * BT : BT;\n"
        "            block_map[3 * nb + 0] = (int32_t)e;\n"
        "            block_map[3 * nb + 1] = (int32_t)(offsets[e] + i * BT);",
        "const int64_t rag = counts[e] - (tiles - 1) * BT;\n"
        "            const int64_t rows = i == 0 ? rag : BT;\n"
        "            block_map[3 * nb + 0] = (int32_t)e;\n"
        "            block_map[3 * nb + 1] = (int32_t)(offsets[e] + (i == 0 ? 0 : rag + (i - 1) * BT));"),
    "nibble_order_swapped": ("(4 * (kk % 2))", "(4 * (1 - kk % 2))"),
    "group_index_wrong": ("scale[n * (K / G) + kk / G]", "scale[n * (K / G) + kk / (2 * G)]"),
    "silu_sign": ("return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    "dropped_first_term": ("for (int64_t kk = 0; kk < d; ++kk) {\n            g +=",
                           "for (int64_t kk = 1; kk < d; ++kk) {\n            g +="),
    "down_transposed": ("acc += Wd[m * f + n] * h[n];", "acc += Wd[n * d + m] * h[n];"),
    "combine_first_slot_only": ("o[(int64_t)pos[t * k + j] * d + m]", "o[(int64_t)pos[t * k] * d + m]"),
    "token_path_overwrites": ("y[s * d + m] += rw[j] * acc;", "y[s * d + m] = rw[j] * acc;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, "mutation site not found: " + name
    mutated = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so_path), str(c_path), "-lm"])
    cdll = oracle.configure(ctypes.CDLL(str(so_path)))
    caught = []
    with oracle.using_library(cdll):
        for check in oc.ALL_CHECKS:
            try:
                check(oracle)
            except AssertionError:
                caught.append(check.__name__)
                break
    assert caught, "no pin caught the planted mistake " + name
