"""Planted mistakes in the oracle (CPU only) must each fail at least one pin.

Every mutant below is a copy of ``oracle/dlrm_oracle.c`` with one plausible
mistake -- a dropped term, a wrong sign, index or operand, a transposed layout,
a missing check -- compiled with the oracle's flags into a temporary library.
The pins of ``oracle_pins.py`` then run against it in a child process (a
mutant may write out of bounds), which must report at least one failure. The
unmodified source, compiled the same way, must pass every pin.
"""
import os
import subprocess
import sys

import pytest

import oracle

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

MUTANTS = {
    "pooled_drops_running_sum": [("acc = acc + w;", "acc = w;")],
    "pooled_wrong_sign": [("acc = acc + w;", "acc = acc - w;")],
    "pooled_skips_first_entry": [("for (int64_t t = s; t < e; ++t) {\n                    float w",
                                  "for (int64_t t = s + 1; t < e; ++t) {\n                    float w")],
    "pooled_layout_transposed": [("int64_t o = ((int64_t)b * F + k) * D + d;",
                                  "int64_t o = ((int64_t)k * B + b) * D + d;")],
    "pooled_all_tables_use_table0_indices": [("indices ? indices + (int64_t)k * seg : NULL",
                                              "indices")],
    "pooled_all_tables_use_weight0": [("const float* W = weights[k];",
                                       "const float* W = weights[0];")],
    "last_bag_ignores_segment_end": [("(int64_t)offsets[(int64_t)k * B + b + 1] : seg;",
                                      "(int64_t)offsets[(int64_t)k * B + b + 1] : s + L;")],
    "offsets_order_unchecked": [("if (s < 0 || s > e || e > seg)", "if (s < 0 || e > seg)")],
    "index_bound_off_by_one": [
        ("int32_t r = indices[(int64_t)k * seg + t];\n            if (r < 0 || (int64_t)r >= rows[k])",
         "int32_t r = indices[(int64_t)k * seg + t];\n            if (r < 0 || (int64_t)r > rows[k])")],
    "general_index_bound_off_by_one": [
        ("int32_t r = indices[(int64_t)k * T + t];\n                if (r < 0 || (int64_t)r >= rows[k])",
         "int32_t r = indices[(int64_t)k * T + t];\n                if (r < 0 || (int64_t)r > rows[k])")],
    "dot_wrong_operand": [("(double)a[d] * (double)b[d]", "(double)a[d] * (double)a[d]")],
    "dot_drops_first_term": [("for (int d = 0; d < D; ++d) {\n        double t",
                              "for (int d = 1; d < D; ++d) {\n        double t")],
    "dot_accumulates_in_float": [("        double t = (double)a[d] * (double)b[d];\n        s += t;",
                                  "        double t = (double)a[d] * (double)b[d];\n"
                                  "        s = (double)((float)s + (float)t);")],
    "dot_bound_loses_the_absolute_value": [("m += (t < 0.0) ? -t : t;", "m += t;")],
    "dot_stores_abs_sum": [("z[p] = (float)s;", "z[p] = (float)m;")],
    "features_in_reverse_table_order": [("emb + ((int64_t)b * F + (i - 1)) * D;",
                                         "emb + ((int64_t)b * F + (F - i)) * D;")],
    "pair_list_transposed": [("if (pi) pi[p] = i;", "if (pi) pi[p] = j;"),
                             ("if (pj) pj[p] = j;", "if (pj) pj[p] = i;")],
    "pairs_include_diagonal": [("for (int j = 0; j < i; ++j) {\n                const float* vj",
                                "for (int j = 0; j <= i; ++j) {\n                const float* vj")],
    "concat_drops_dense": [("row[d] = dense[(int64_t)b * D + d];", "row[d] = 0.0f;")],
    "bf16_widened_with_wrong_shift": [("((uint32_t)h) << 16", "((uint32_t)h) << 15")],
    "weighted_sum_drops_weight": [("acc = fmaf(wk[t], x, acc);", "acc = acc + x;")],
    "weighted_sum_rounds_the_product_first": [("acc = fmaf(wk[t], x, acc);",
                                               "acc = acc + wk[t] * x;")],
    "mean_multiplies_by_reciprocal": [("acc = acc / (float)(e - s);",
                                       "acc = acc * (1.0f / (float)(e - s));")],
    "weighted_sum_uses_first_weight": [("acc = fmaf(wk[t], x, acc);",
                                        "acc = fmaf(wk[s], x, acc);")],
    "mean_divides_by_count_plus_one": [("acc = acc / (float)(e - s);",
                                        "acc = acc / (float)(e - s + 1);")],
    "max_keeps_the_minimum": [("((x > acc) ? x : acc)", "((x < acc) ? x : acc)")],
    "max_ties_take_the_later_entry": [("acc = (t == s) ? x : ((x > acc) ? x : acc);",
                                       "acc = (t == s) ? x : ((x >= acc) ? x : acc);")],
    "mean_of_empty_bag_divides_by_zero": [("if (mode == ORACLE_POOL_MEAN && e > s) acc",
                                           "if (mode == ORACLE_POOL_MEAN) acc")],
    "max_starts_from_zero": [("acc = (t == s) ? x : ((x > acc) ? x : acc);",
                              "acc = (x > acc) ? x : acc;")],
    "last_offset_ignored": [("(ilo || b + 1 < B) ? (int64_t)offsets[(int64_t)k * row + b + 1]",
                             "(b + 1 < B) ? (int64_t)offsets[(int64_t)k * row + b + 1]")],
    "linear_weight_transposed": [("(double)bf16_bits_to_f32(wn[k]);", "(double)bf16_bits_to_f32(w[k * ldw + n]);")],
    "linear_hi_part_reads_lo_weights": [("(double)bf16_bits_to_f32(wn[k_lo + k]);",
                                         "(double)bf16_bits_to_f32(wn[k]);")],
    "linear_bias_subtracted": [("s += (double)bias[n];", "s -= (double)bias[n];")],
    "linear_relu_after_sigmoid_swapped": [("if (act == 1) y = (s > 0.0) ? s : 0.0;",
                                           "if (act == 2) y = (s > 0.0) ? s : 0.0;")],
    "linear_sigmoid_sign": [("y = 1.0 / (1.0 + exp(-s));", "y = 1.0 / (1.0 + exp(s));")],
    "linear_a_row_pitch_ignored": [("bf16_bits_to_f32(a_lo[m * lda_lo + k])",
                                    "bf16_bits_to_f32(a_lo[m * k_lo + k])")],
    "linear_f32a_activation_narrowed": [
        ("const double t = (double)a_lo[m * lda_lo + k] * weight_at(w, w_bf16, n * ldw + k);",
         "const double t = (double)(float)((double)(int)(a_lo[m * lda_lo + k] * 256.0f) / 256.0)"
         " * weight_at(w, w_bf16, n * ldw + k);")],
    "linear_f32a_product_rounded_to_f32": [
        ("const double t = (double)a_lo[m * lda_lo + k] * weight_at(w, w_bf16, n * ldw + k);",
         "const double t = (double)(float)((double)a_lo[m * lda_lo + k] *"
         " weight_at(w, w_bf16, n * ldw + k));")],
    "linear_f32a_hi_part_reads_lo_weights": [("weight_at(w, w_bf16, n * ldw + k_lo + k)",
                                               "weight_at(w, w_bf16, n * ldw + k)")],
    "linear_f32a_weight_transposed": [("weight_at(w, w_bf16, n * ldw + k);",
                                        "weight_at(w, w_bf16, k * ldw + n);")],
    "linear_f32a_bf16_weights_read_as_integers": [
        ("return (double)bf16_bits_to_f32(((const uint16_t*)w)[i]);",
         "return (double)((const uint16_t*)w)[i];")],
    "linear_f32a_a_row_pitch_ignored": [("(double)a_lo[m * lda_lo + k]",
                                         "(double)a_lo[m * k_lo + k]")],
    "general_pooling_table_layout_transposed": [
        ("out[((int64_t)b * F + k) * D + d] = acc;", "out[((int64_t)k * B + b) * D + d] = acc;")],
}

_RUNNER = (
    "import sys; sys.path[:0] = [{root!r}, {tests!r}]\n"
    "import oracle, oracle_pins\n"
    "sys.exit(min(100, oracle_pins.run_all(oracle.Oracle({lib!r}))))\n"
)


def _build_and_run(tmp_path, name, edits):
    with open(oracle.SOURCE) as fh:
        src = fh.read()
    for old, new in edits:
        assert src.count(old) == 1, f"mutant {name}: pattern must occur exactly once: {old!r}"
        src = src.replace(old, new)
    csrc = tmp_path / f"{name}.c"
    csrc.write_text(src)
    lib = str(tmp_path / f"lib{name}.so")
    oracle.compile_source(str(csrc), lib)
    code = _RUNNER.format(root=ROOT, tests=TESTS, lib=lib)
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=300)


def test_unmutated_copy_passes_every_pin(tmp_path):
    r = _build_and_run(tmp_path, "control", [])
    assert r.returncode == 0, r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(tmp_path, name):
    r = _build_and_run(tmp_path, name, MUTANTS[name])
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stderr[-2000:]}"
