"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check
that the pins catch every one of them."""
import os
import shutil
import subprocess
import tempfile
import types

import pytest

import oracle
import tests.test_oracle_pins as pins
from tests.conftest import read_golden

MUTATIONS = {
    "dropped_half_in_rounding": ("float shifted = ratio + 0.5f;", "float shifted = ratio;"),
    "scale_over_16": ("(hi - lo) / (float)levels", "(hi - lo) / (float)(levels + 1)"),
    "lsb_first_planes": ("pc[(bits - 1 - p) * n_words + j / 32] |=", "pc[p * n_words + j / 32] |="),
    "variance_missing_square": ("double sc2 = sc * sc;", "double sc2 = sc;"),
    "importance_uses_abs_q": ("float qq = qc * qc;", "float qq = fabsf(qc);"),
    "plan_ascending_importance": ("if (a->key > b->key) return -1;\n    if (a->key < b->key) return 1;",
                                  "if (a->key < b->key) return -1;\n    if (a->key > b->key) return 1;"),
    "plan_cap_3_bits": ("take = left < bits ? left : bits;", "take = left < 3 ? left : 3;"),
    "bin_low_edge_not_middle": ("(double)(width - 1) / 2.0", "0.0"),
    "planes_read_lsb_first": ("u = (u << 1) | (int)((word >> (j % 32)) & 1u);",
                              "u = u | (int)(((word >> (j % 32)) & 1u) << slot);"),
    "topk_ties_to_higher_index": ("return (a->j < b->j) ? -1 : (a->j > b->j);",
                                  "return (a->j > b->j) ? -1 : (a->j < b->j);"),
    "union_takes_min": ("if (t[g * d + c] > m) m = t[g * d + c];", "if (g == 0) m = t[g * d + c];"),
    "append_lsb_first": ("if ((v >> p) & 1)\n                        pc[(bits - 1 - p) * n_words",
                         "if ((v >> p) & 1)\n                        pc[p * n_words"),
    "append_ignores_min": ("float diff = x - lo;", "float diff = x;"),
    "append_variance_old_count": ("const int64_t nn = n + m;", "const int64_t nn = n;"),
    "append_no_high_clamp_count": ("out_of_range = level < 0.0f || level > (float)levels;",
                                   "out_of_range = level < 0.0f;"),
    "attention_no_max_shift": ("const double p = exp(logit[i] - mx);", "const double p = exp(logit[i]);"),
    "attention_unscaled_logits": ("logit[i] = scale * acc;", "logit[i] = acc;"),
    "marginal_gain_ignores_depth": ("const float gain = w[c] * (1.0f / (float)(1 << (2 * t[c])));",
                                    "const float gain = w[c];"),
    "marginal_gain_halves": ("(float)(1 << (2 * t[c]))", "(float)(1 << t[c])"),
    "merge_ignores_offset": ("items[s * k_s + i].j = offset[s] + idx[s * k_s + i];",
                             "items[s * k_s + i].j = idx[s * k_s + i];"),
    "merge_output_not_index_ordered": ("while (p >= 0 && items[p].j > x.j)", "while (0)"),
    "quantize_levels_stay_15": ("const int levels = (1 << bits) - 1;", "const int levels = 15;"),
    "plan_cap_stays_4_bits": ("take = left < bits ? left : bits;", "take = left < 4 ? left : 4;"),
    "fixed_plan_reads_4_bits": ("(uint8_t)(i < r ? bits : 0)", "(uint8_t)(i < r ? 4 : 0)"),
    "unpack_reads_4_slots": ("for (int p = 0; p < bits; ++p)\n                    v |=",
                             "for (int p = 0; p < bits && p < 4; ++p)\n                    v |="),
    "midpoint_of_4bit_bins": ("double level = (double)(width * u) + (double)(width - 1) / 2.0;",
                              "double level = (double)(width * u) + (double)((width < 16 ? width : 16) - 1) / 2.0;"),
    "blocked_sigma2_no_between_block_term": (
        "M2 = M2 + m2_b + (delta * delta) * ((N * nbd) / Nn);", "M2 = M2 + m2_b;"),
    "blocked_sigma2_mean_ignores_min": ("const double mean_b = (double)mn[i] + sc *",
                                        "const double mean_b = 0.0 + sc *"),
    "attention_unnormalised": ("for (int64_t c = 0; c < d; ++c) out[c] /= denom;",
                               "for (int64_t c = 0; c < d; ++c) out[c] /= (double)cnt;"),
    "abs_sum_takes_abs_of_the_sum": (
        "acc += fabs((double)bf16_value(q_bf16[c]) *\n"
        "                        fo_coarse_midpoint(mn[c], scale[c], tc, u, (int)bits));\n"
        "        }\n        a[j] = acc;",
        "acc += ((double)bf16_value(q_bf16[c]) *\n"
        "                        fo_coarse_midpoint(mn[c], scale[c], tc, u, (int)bits));\n"
        "        }\n        a[j] = fabs(acc);"),
    "abs_sum_reads_every_plane": (
        "int64_t n, int64_t n_words, double *a)\n{\n    if (!fo_bits_ok(bits)) return FO_ERR_ARG;\n"
        "    for (int64_t j = 0; j < n; ++j) {\n        double acc = 0.0;\n"
        "        for (int64_t c = 0; c < d; ++c) {\n            int tc = t[c];\n"
        "            if (tc < 0 || tc > bits) return FO_ERR_ARG;\n            int u = 0;\n"
        "            for (int slot = 0; slot < tc; ++slot) {",
        "int64_t n, int64_t n_words, double *a)\n{\n    if (!fo_bits_ok(bits)) return FO_ERR_ARG;\n"
        "    for (int64_t j = 0; j < n; ++j) {\n        double acc = 0.0;\n"
        "        for (int64_t c = 0; c < d; ++c) {\n            int tc = t[c];\n"
        "            if (tc < 0 || tc > bits) return FO_ERR_ARG;\n            int u = 0;\n"
        "            for (int slot = 0; slot < bits; ++slot) {"),
    "exact_scores_transposed_keys": ("(double)keys_h[j * d + c]", "(double)keys_h[c * n + j]"),
    "plan_ties_to_higher_channel": ("return (a->c < b->c) ? -1 : (a->c > b->c);",
                                    "return (a->c > b->c) ? -1 : (a->c < b->c);"),
    "plan_leftover_skips_zero_importance": ("        if (left > 0) {\n            take = left < bits",
                                            "        if (left > 0 && order[i].key > 0.0f) {\n"
                                            "            take = left < bits"),
    "bytes_per_plane_in_words": ("(uint64_t)t[c] * (uint64_t)n_words * 4u", "(uint64_t)t[c] * (uint64_t)n_words"),
    "variance_over_n_minus_1": ("double nn = (double)n * (double)n;",
                                "double nn = (double)n * (double)(n - 1);"),
    "score_skips_zero_depth_channels": (
        "            acc += (double)bf16_value(q_bf16[c]) *\n                   fo_coarse_midpoint",
        "            if (tc > 0) acc += (double)bf16_value(q_bf16[c]) *\n                   fo_coarse_midpoint"),
    "importance_ignores_variance": ("float wc = qq * sigma2[c];", "float wc = qq;"),
    "marginal_gain_ties_to_higher_channel": ("if (best < 0 || gain > best_gain) {",
                                             "if (best < 0 || gain >= best_gain) {"),
    "topk_keeps_lowest_scores": ("if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
                                 "if (a->s < b->s) return -1;\n    if (a->s > b->s) return 1;"),
}

PIN_TESTS = [
    lambda: pins.test_quantize_hand_worked(read_golden),
    pins.test_quantize_error_bound_and_extremes,
    pins.test_sigma2_matches_variance_of_dequantised_keys,
    lambda: pins.test_plane_layout_hand_worked(read_golden),
    pins.test_importance_values,
    lambda: pins.test_plan_hand_worked(read_golden),
    lambda: pins.test_plan_is_optimal_by_brute_force_small(3),
    lambda: pins.test_fixed_plan_hand_worked(read_golden),
    pins.test_union_and_bytes,
    lambda: pins.test_coarse_bin_midpoint_hand_worked(read_golden),
    pins.test_reading_t_planes_equals_requantising_to_t_bits,
    lambda: pins.test_topk_hand_worked(read_golden),
    lambda: pins.test_append_in_range_equals_repacking_everything(127, 129),
    pins.test_append_clamps_out_of_range_keys_to_the_end_levels,
    pins.test_append_keeps_sigma2_the_variance_of_the_stored_keys,
    pins.test_attention_over_every_key_is_dense_attention,
    pins.test_attention_special_cases,
    pins.test_marginal_plan_spreads_uniform_importance_round_robin,
    pins.test_marginal_plan_hand_worked,
    lambda: pins.test_merging_shard_topks_is_the_topk_of_all_keys(3, 999, 64),
    pins.test_quantize_8bit_hand_worked,
    pins.test_quantize_8bit_error_bound_and_extremes,
    pins.test_plane_layout_8bit_hand_worked,
    lambda: pins.test_planes_8bit_round_trip_and_size(1000),
    pins.test_coarse_bin_8bit_is_mean_of_its_fine_levels,
    lambda: pins.test_plan_8bit_is_optimal_by_brute_force(2),
    pins.test_fixed_plan_8bit_reads_whole_channels,
    pins.test_append_8bit_in_range_equals_repacking_and_clamps,
    pins.test_blocked_sigma2_is_the_variance_of_all_dequantised_keys,
    pins.test_blocks_as_large_as_the_keys_are_the_global_quantiser,
    lambda: pins.test_score_and_absolute_sum_hand_worked(read_golden),
    lambda: pins.test_exact_scores_hand_worked(read_golden),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found"
    tmp = tempfile.mkdtemp()
    try:
        csrc = os.path.join(tmp, "mut.c")
        so = os.path.join(tmp, "mut.so")
        open(csrc, "w").write(src.replace(old, new, 1))   # first occurrence
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC",
                               "-shared", "-o", so, csrc, "-lm"])
        monkeypatch.setattr(oracle, "_LIB_PATH", so)
        monkeypatch.setattr(oracle, "build", lambda force=False: so)
        monkeypatch.setattr(oracle, "_lib", None)
        caught = 0
        for fn in PIN_TESTS:
            try:
                fn()
            except (AssertionError, ValueError):
                caught += 1
        assert caught >= 1, f"no pin caught mutation {name}"
    finally:
        shutil.rmtree(tmp)


# Planted mistakes in the Python side of the oracle (the session-level steps
# around the C routines: per-head plans, the GQA union, bytes, block ranges,
# appends of whole blocks, the per-head absolute sum, the error metric).
PY_MUTATIONS = {
    "session_plan_reads_another_heads_variance": ("        h = q // group\n", "        h = q % group\n"),
    "session_union_over_the_wrong_queries": ("union(t[h * group:(h + 1) * group])",
                                             "union(t[h:h + group])"),
    "session_head_bytes_from_a_query_plan": ('[plan_bytes(T[h], index["n_words"]) for h in range(H)]',
                                             '[plan_bytes(t[h], index["n_words"]) for h in range(H)]'),
    "blocked_index_quantises_the_first_keys_for_every_block": (
        "quantize(keys[:, j0:j1], bits)", "quantize(keys[:, :j1 - j0], bits)"),
    "append_blocks_overwrites_the_first_blocks": ("b = (n + i0) // block", "b = i0 // block"),
    "append_blocks_variance_of_the_old_key_count": ('index["s2"][h], n + m, block)',
                                                    'index["s2"][h], n, block)'),
    "head_blocks_use_the_first_blocks_scales": ('index["mn"][h, b], index["scale"][h, b]))',
                                                'index["mn"][h, 0], index["scale"][h, 0]))'),
    "score_head_ignores_absolute": ("fn = score_abs_planes if absolute else score_planes",
                                    "fn = score_planes"),
    "attention_error_not_relative": ("np.linalg.norm(o - o_exact) / np.linalg.norm(o_exact)",
                                     "np.linalg.norm(o - o_exact)"),
    "plane_rows_of_32_keys": ("((n + 127) // 128) * 4", "(n + 31) // 32"),
}

PY_PIN_TESTS = [
    pins.test_union_and_bytes,
    pins.test_plans_of_a_blocked_index_use_its_channel_variance,
    pins.test_blocked_append_of_whole_blocks_equals_packing_everything,
    pins.test_blocked_scores_full_zero_and_prefix_depths,
    pins.test_blocked_sigma2_is_the_variance_of_all_dequantised_keys,
    pins.test_absolute_scores_bound_the_scores_and_equal_them_when_no_term_is_negative,
    pins.test_attention_error_metric,
    lambda: pins.test_planes_round_trip_and_padding(1),
    pins.test_tiny_workload_planted_keys_rank_high,
]


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_pins_catch_planted_mistake_in_the_python_oracle(name, monkeypatch):
    old, new = PY_MUTATIONS[name]
    src = open(oracle.__file__).read()
    assert src.count(old) == 1, "mutation anchor not found once"
    mutant = types.ModuleType("oracle_mutant")
    mutant.__file__ = oracle.__file__
    exec(compile(src.replace(old, new), oracle.__file__, "exec"), mutant.__dict__)
    monkeypatch.setattr(pins, "oracle", mutant)
    caught = 0
    for fn in PY_PIN_TESTS:
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin caught mutation {name}"
