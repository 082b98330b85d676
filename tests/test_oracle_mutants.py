"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Each mutant rewrites one plausible slip into a private copy of the oracle's C
source (a dropped term, a wrong sign, a wrong index, a transposed operand, a
wrong rounding, a non-strict threshold ...), compiles it to a temporary
library, and runs the pins against it. A mutant that no pin catches means the
pins leave that part of the oracle unchecked.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "sgq_oracle.c")

MUTANTS = {
    "drop_zero_point": ("double w = sv * ((double)q[(size_t)n * K + k] - zv);",
                        "double w = sv * ((double)q[(size_t)n * K + k]);"),
    "zero_point_sign": ("- zv);", "+ zv);"),
    "group_index": ("int grp = k / g;", "int grp = (k / g + 1) % G;"),
    "transposed_codes": ("q[(size_t)n * K + k]", "q[(size_t)k * N + n]"),
    "threshold_not_strict": ("if (a > (double)t[b])", "if (a >= (double)t[b])"),
    "zero_floor": ("zv = clamp15(nearbyint(-lo / sv));", "zv = clamp15(floor(-lo / sv));"),
    "code_floor": ("double c = clamp15(nearbyint(w / sv) + zv);",
                   "double c = clamp15(floor(w / sv) + zv);"),
    "scale_over_16": ("(hi - lo) / 15.0", "(hi - lo) / 16.0"),
    "range_without_zero": ("double lo = 0.0, hi = 0.0;", "double lo = INFINITY, hi = -INFINITY;"),
    "drop_last_active": ("for (int i = 0; i < count; ++i) {\n        int k = idx[i];",
                         "for (int i = 0; i < count - 1; ++i) {\n        int k = idx[i];"),
    "nibble_order": ("(uint8_t)(lo | (hi << 4))", "(uint8_t)(hi | (lo << 4))"),
    "ties_away_from_zero": ("return nearbyint(a / quantum) * quantum;",
                            "return round(a / quantum) * quantum;"),
    "bf16_exponent": ("e - 127 - 7", "e - 127 - 6"),
    "half_subnormal": ("ldexp((double)m, -24)", "ldexp((double)m, -25)"),
    "silu_sign": ("exp(-gv)", "exp(gv)"),
    "union_last_row_only": ("for (int b = 0; b < B; ++b) {\n            double a",
                            "for (int b = B - 1; b < B; ++b) {\n            double a"),
    "sumabs_signed": ("acc_abs += fabs(p);", "acc_abs += p;"),
    "mask_bit_order": ("mask[idx[i] / 32] |= 1u << (idx[i] % 32);",
                       "mask[idx[i] / 32] |= 1u << (31 - idx[i] % 32);"),
    "mask_word_index": ("mask[idx[i] / 32] |= 1u << (idx[i] % 32);",
                        "mask[idx[i] / 8 % ((K + 31) / 32)] |= 1u << (idx[i] % 32);"),
    "nm_ties_to_higher": ("if (first < 0 || e[i] > e[first]) {",
                          "if (first < 0 || e[i] >= e[first]) {"),
    "nm_energy_abs": ("                    acc += w * w;\n",
                      "                    acc += fabs(w);\n"),
    "nm_keep_nibble_order": ("(uint8_t)(keep[(size_t)grp * (N / 4) + 2 * jj] |",
                             "(uint8_t)(keep[(size_t)grp * (N / 4) + 2 * jj + 1] |"),
    "nm_slot_order": ("qweight[(size_t)k * (N / 4) + j] = (uint8_t)(c0 | (c1 << 4));",
                      "qweight[(size_t)k * (N / 4) + j] = (uint8_t)(c1 | (c0 << 4));"),
    "act_mul_drops_up": ("double hv = oracle_act(gate[i], act) * up[i];",
                         "double hv = oracle_act(gate[i], act);"),
    "threads_skip_last_output": ("for (long long o = 0; o < total; ++o)",
                                 "for (long long o = 0; o < total - 1; ++o)"),
    "threads_batch_forgotten": ("long long total = (long long)B * N;", "long long total = N;"),
    "act_mul_swapped": ("double hv = oracle_act(gate[i], act) * up[i];",
                        "double hv = oracle_act(up[i], act) * gate[i];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    orig, repl = MUTANTS[name]
    src = open(SRC).read()
    assert orig in src, f"mutation site for {name} no longer in the oracle"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(orig, repl))
    lib = oracle.load(oracle.build(force=True, src=str(mpath), out=str(tmp_path / "libmut.so")))
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            return
        except oracle.OracleError:
            return
    pytest.fail(f"no pin catches mutant {name}")
