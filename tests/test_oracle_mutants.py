"""Planted mistakes: each copy of oracle.c below carries one plausible bug
(a dropped term, a wrong sign, index or operand, a misplaced floor, a broken
tie rule or rounding, in the fp path, in int8 coding and scoring and
in the in-batch softmax). Every copy must fail at least one pin; a copy that
passes them all would show a gap in the pins. CPU only; the copies are built
in a temporary directory and never touch the real oracle."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "dropped_square": ("ss += x * x;", "ss += x;"),
    "eps_added_to_norm": ("sqrt(ss > ORACLE_EPS ? ss : ORACLE_EPS)", "(sqrt(ss) + ORACLE_EPS)"),
    "eps_floor_ignored": ("ss > ORACLE_EPS ? ss : ORACLE_EPS", "ss"),
    "multiply_by_norm": ("x / norm", "x * norm"),
    "ascending_sort": ("if (a->s > b->s)\n        return -1;\n    if (a->s < b->s)\n        return 1;",
                       "if (a->s > b->s)\n        return 1;\n    if (a->s < b->s)\n        return -1;"),
    "higher_id_wins_ties": ("if (a->id < b->id)\n        return -1;\n    if (a->id > b->id)\n        return 1;",
                            "if (a->id < b->id)\n        return 1;\n    if (a->id > b->id)\n        return -1;"),
    "tau_multiplies": ("return dot / tau;", "return dot * tau;"),
    "fused_norm_multiplies": ("dot = dot / norms[j];", "dot = dot * norms[j];"),
    "mask_bit_index": ("(j & 31)", "(j & 15)"),
    "mask_word_index": ("exclude[j >> 5]", "exclude[j >> 6]"),
    "query_coordinates_reversed": ("load_elem(q, q_dtype, qrow * (int64_t)d + i)",
                                   "load_elem(q, q_dtype, qrow * (int64_t)d + (d - 1 - i))"),
    "id_after_compaction": ("pairs[m].id = j;", "pairs[m].id = m;"),
    "bf16_truncates": ("rint(ax / quantum)", "floor(ax / quantum)"),
    "bf16_one_bit_short": ("ldexp(1.0, lead - 7)", "ldexp(1.0, lead - 6)"),
    "bf16_load_shift": ("(uint32_t)h << 16", "(uint32_t)h << 15"),
    "pad_score_zero": ("out_scores[qi * k + r] = -INFINITY;", "out_scores[qi * k + r] = 0.0;"),
    # int8 coding and scoring
    "q8_scale_over_128": ("maxabs / 127.0f", "maxabs / 128.0f"),
    "q8_round_half_away": ("rintf(w / us)", "roundf(w / us)"),
    "q8_truncate": ("rintf(w / us)", "truncf(w / us)"),
    "q8_scale_floor_missing": ("if (us < ORACLE_Q8_FLOOR)\n            us = ORACLE_Q8_FLOOR;", ""),
    "q8_not_normalised": ("float w = normalise ? (float)(x / norm) : (float)x;", "float w = (float)x;"),
    "q8_row_scale_dropped": ("dot = dot * (double)qscales[qrow] * (double)vscales[j];",
                             "dot = dot * (double)qscales[qrow];"),
    "q8_code_sign_lost": ("codes[j * (int64_t)d + i] = (int8_t)r;", "codes[j * (int64_t)d + i] = (int8_t)fabsf(r);"),
    # in-batch sampled softmax
    "logq_added": ("l[j] -= logq[j];", "l[j] += logq[j];"),
    "logq_skips_positive": ("            if (logq)\n                l[j] -= logq[j];",
                            "            if (logq && j != i)\n                l[j] -= logq[j];"),
    "hit_masks_positive": ("if (item_ids && j != i && item_ids[j] == item_ids[i])",
                           "if (item_ids && item_ids[j] == item_ids[i])"),
    "hit_compares_index": ("item_ids[j] == item_ids[i])", "item_ids[j] == (int64_t)i)"),
    "invalid_column_kept": ("    if (valid && !valid[j])\n        return 0;\n", ""),
    "invalid_row_counted": ("loss[i] = (!valid || valid[i]) ? lse[i] - l[i] : 0.0;", "loss[i] = lse[i] - l[i];"),
    "mean_over_all_rows": ("total / (double)rows", "total / (double)b"),
    "max_not_factored_back": ("m + log(sum)", "log(sum)"),
    "numerator_first_column": ("lse[i] - l[i]", "lse[i] - l[0]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    path_c = tmp_path / f"{name}.c"
    path_c.write_text(src.replace(old, new))
    lib = oracle.OracleLib(oracle.build(force=True, src=str(path_c), out=str(tmp_path / f"{name}.so")))
    failures = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(lib)
        except AssertionError:
            failures.append(check.__name__)
    assert failures, f"planted mistake {name!r} passed every pin"
