"""Planted mistakes in copies of the oracle must fail at least one pin.

Each mutant is the oracle's C source with one plausible slip (a dropped term,
a wrong sign or index, a transposed operand, a missed mask), compiled to a
temporary library.  The real oracle passes every pin (test_oracle_pins.py);
these show the pins are strong enough to catch each slip.
"""
import os
import shutil

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "qsa_oracle.c")

MUTANTS = {
    "lse_without_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "score_sign": ("s[j] = scale * dot;", "s[j] = -scale * dot;"),
    "kv_head_index": ("const int64_t g = h / G;", "const int64_t g = h % a->num_kv_heads;"),
    "scores_from_v": ("const uint16_t* kr = a->k + sel[j]", "const uint16_t* kr = a->v + sel[j]"),
    "no_normalisation": ("for (int64_t d = 0; d < D; ++d) out_row[d] /= l;", ""),
    "default_scale_1_over_d": ("1.0 / sqrt((double)D)", "1.0 / (double)D"),
    "ignores_n_valid": ("if (nv < n_list) n_list = nv;", ""),
    "drops_first_entry": ("for (int64_t j = 0; j < n_list; ++j) {", "for (int64_t j = 1; j < n_list; ++j) {"),
    "empty_lse_zero": ("*lse_out = -INFINITY;", "*lse_out = 0.0;"),
    "widening_shift": ("((uint32_t)bits) << 16", "((uint32_t)bits) << 15"),
    "idx_head_stride_dropped": ("g * a->idx_stride_head", "0 * a->idx_stride_head"),
    "sum_before_exp": ("{ s[j] = exp(s[j] - m); l += s[j]; }", "{ l += s[j]; s[j] = exp(s[j] - m); }"),
    "block_offset_dropped": ("const int64_t slot = id * bs + r;", "const int64_t slot = id * bs;"),
    "last_slot_ignored": ("if (slot >= a->num_slots || slot > limit) continue;", "if (slot >= a->num_slots) continue;"),
    "v_head_stride_dropped": ("const uint16_t* vr = a->v + sel[j] * a->kv_stride_slot + g * a->kv_stride_head;",
                              "const uint16_t* vr = a->v + sel[j] * a->kv_stride_slot;"),
    "indexer_head_dropped": ("for (int64_t h = 0; h < a->num_heads; ++h) {",
                             "for (int64_t h = 1; h < a->num_heads; ++h) {"),
    "indexer_partial_block": ("int64_t hi = ((int64_t)a->positions[t] + 1) / bs;",
                              "int64_t hi = ((int64_t)a->positions[t] + bs) / bs;"),
    "indexer_sequence_start_ignored": ("int64_t lo = a->seq_start[t] / bs;", "int64_t lo = 0;"),
    "indexer_key_row_of_token": ("const uint16_t* kr = a->k + b * a->k_stride_block;",
                                 "const uint16_t* kr = a->k + t * a->k_stride_block;"),
    "topk_keeps_lowest": ("if (a->score > b->score) return -1;\n  if (a->score < b->score) return 1;",
                          "if (a->score < b->score) return -1;\n  if (a->score > b->score) return 1;"),
    "topk_ties_to_larger_block": ("return (a->block > b->block) - (a->block < b->block);",
                                  "return (a->block < b->block) - (a->block > b->block);"),
    "e4m3_exponent_bias": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_as_normal": ("e == 0 ? ldexp((double)m, -9)", "e == 0 ? ldexp(1.0 + m / 8.0, -7)"),
    "fp8_k_scale_dropped": ("(qsa_oracle_e4m3_to_double(kb[d]) * a->k_scale)", "qsa_oracle_e4m3_to_double(kb[d])"),
    "fp8_v_scaled_by_k_scale": ("(qsa_oracle_e4m3_to_double(vb[d]) * a->v_scale)",
                                "(qsa_oracle_e4m3_to_double(vb[d]) * a->k_scale)"),
    "topk_tail_always": ("if (append_tail && ((int64_t)a->positions[t] + 1) % bs != 0)", "if (append_tail)"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_dir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    d = mutant_dir / name
    d.mkdir()
    msrc = d / "qsa_oracle.c"
    msrc.write_text(src.replace(old, new))
    shutil.copy(os.path.join(os.path.dirname(SRC), "qsa_oracle.h"), d / "qsa_oracle.h")
    lib = oracle.build(force=True, src=str(msrc), out=str(d / "libmutant.so"))
    orc = oracle.Oracle(lib)
    failed = []
    for check in P.ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"
