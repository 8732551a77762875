"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source (on the CPU only),
compiles it, points the oracle wrapper at the broken library and runs the pins that cover the
routine.  At least one pin must fail for every planted mistake; the real library is restored
afterwards.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild

from . import test_oracle_accept as ta
from . import test_oracle_draft_layer as tdl
from . import test_oracle_attention as tt
from . import test_oracle_text_attention as tx
from . import test_oracle_topk_hsr as tk

ATTN = [tt.test_golden_attention_tiny, lambda: tt.test_verify_matches_torch_sdpa("f32"),
        tt.test_verify_gamma0_equals_single_token_decode, tt.test_verify_zero_keys_give_running_mean]
TEXT = [tt.test_golden_text_anchored_tiny, lambda: tt.test_text_anchored_window_crossing_the_visual_span(12),
        tt.test_text_anchored_wide_window_equals_dense_without_visual_span]
SPARSE = [tt.test_sparse_matches_torch_with_explicit_set_mask,
          tt.test_sparse_with_all_candidates_equals_dense]
TOPK = [tk.test_golden_topk_tiny, lambda: tk.test_topk_brute_force_over_all_subsets(0, 3),
        tk.test_topk_duplicated_keys_tie_to_lower_positions]
HSR = [tk.test_hsr_matches_torch_fp64_matmul, tk.test_hsr_concatenation_order]
TEXT_ATTN = [tx.test_golden_text_attention_tiny, lambda: tx.test_scores_over_every_position_sum_to_one(0),
             lambda: tx.test_scores_equal_mean_attention_output_with_one_hot_values(1, 3),
             tx.test_zero_keys_give_uniform_weights_closed_form,
             tx.test_candidates_beyond_a_rows_causal_limit_get_only_the_later_rows]
DRAFT = [tdl.test_rmsnorm_matches_torch_fp64, tdl.test_rope_equals_complex_rotation,
         tdl.test_layer_input_is_the_hsr_projection_and_zero_projections_pass_it_through,
         tdl.test_layer_attention_is_the_text_anchored_attention_over_the_appended_cache,
         tdl.test_layer_with_zero_norm_weights_has_closed_forms,
         tdl.test_layer_with_zero_input_norm_projects_the_bias_rotated_at_the_row_positions,
         tdl.test_layer_mlp_half_matches_torch_fp64]
GREEDY = [ta.test_golden_accept_greedy_tiny, ta.test_greedy_argmax_ties_nan_and_signed_zero,
          ta.test_greedy_own_argmax_accepts_everything]
SAMPLE = [ta.test_golden_accept_sample_tiny,
          lambda: ta.test_sampling_brute_force_reproduces_target_distribution_gamma1(0),
          ta.test_sampling_brute_force_reproduces_target_distribution_gamma2]

MUTANTS = {
    "scale_1_over_d": ("1.0 / sqrt((double)head_dim)", "1.0 / (double)head_dim", ATTN),
    "causal_off_by_one": ("int64_t limit = kv_len - n_q + i;\n    for (int64_t j = 0; j <= limit; ++j)\n        pos[j] = j;",
                          "int64_t limit = kv_len - n_q + i - 1;\n    for (int64_t j = 0; j <= limit; ++j)\n        pos[j] = j;", ATTN),
    "gqa_modulo_mapping": ("            int g = h / G;\n", "            int g = h % c->h_kv;\n", ATTN),
    "missing_max_shift_denominator": ("den += w;", "den += 1.0;", ATTN),
    "visual_span_inclusive_start": ("if (j >= vb && j < ve)", "if (j > vb && j < ve)", TEXT),
    "window_ends_before_own_position": ("for (int64_t j = limit; j >= 0 && n < W; --j) {",
                                        "for (int64_t j = limit - 1; j >= 0 && n < W; --j) {", TEXT),
    "sparse_tail_starts_one_late": ("int64_t tb = t->tail_begin[b] < 0 ? 0 : t->tail_begin[b];",
                                    "int64_t tb = t->tail_begin[b] < 0 ? 0 : t->tail_begin[b] + 1;", SPARSE),
    "sparse_drops_selection": ("mark[sel[e]] = 1;", "mark[sel[e]] = 0;", SPARSE),
    "topk_ties_to_higher": ("return (x->j < y->j) ? -1 : (x->j > y->j);",
                            "return (x->j > y->j) ? -1 : (x->j < y->j);", TOPK),
    "topk_smallest_scores": ("if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
                             "if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;", TOPK),
    "text_attention_not_causal": ("int64_t limit = kv_len - n_q + i;\n                for (int e = 0; e < d; ++e)",
                                  "int64_t limit = kv_len - 1;\n                for (int e = 0; e < d; ++e)", TEXT_ATTN),
    "text_attention_sum_not_mean_over_heads": ("dst[t] /= (double)G * (double)n_q;",
                                               "dst[t] /= (double)n_q;", TEXT_ATTN),
    "text_attention_first_head_of_group_only": ("for (int h = g * G; h < (g + 1) * G; ++h) {\n            for (int64_t i = 0; i < n_q; ++i) {",
                                                "for (int h = g * G; h < g * G + 1; ++h) {\n            for (int64_t i = 0; i < n_q; ++i) {", TEXT_ATTN),
    "text_attention_unscaled": ("s[j] = scale * dot;", "s[j] = dot;", TEXT_ATTN),
    "text_attention_denominator_from_candidates": ("for (int64_t j = 0; j <= limit; ++j)\n                    den += exp(s[j] - m);",
                                                   "for (int64_t j = cb; j <= limit && j < ce; ++j)\n                    den += exp(s[j] - m);", TEXT_ATTN),
    "rope_rotation_sign": ("v[i] = a * c - b * s;", "v[i] = a * c + b * s;", DRAFT),
    "rope_frequency_exponent": ("pow(theta, -2.0 * (double)i / (double)d)",
                                "pow(theta, -1.0 * (double)i / (double)d)", DRAFT),
    "rmsnorm_sum_not_mean": ("1.0 / sqrt(ss / (double)n + eps)", "1.0 / sqrt(ss + eps)", DRAFT),
    "draft_attention_residual_missing": ("            x2[i] += x[(int64_t)r * D + i];\n",
                                         "            x2[i] += 0.0;\n", DRAFT),
    "draft_silu_as_sigmoid": ("sv[i] = gu[i] / (1.0 + exp(-gu[i])) * gu[F + i];",
                              "sv[i] = 1.0 / (1.0 + exp(-gu[i])) * gu[F + i];", DRAFT),
    "draft_gate_up_swapped": ("sv[i] = gu[i] / (1.0 + exp(-gu[i])) * gu[F + i];",
                              "sv[i] = gu[F + i] / (1.0 + exp(-gu[F + i])) * gu[i];", DRAFT),
    "draft_rope_position_one_late": ("orc_rope(qkv + (int64_t)h * d, d, (double)pos, w->rope_theta);",
                                     "orc_rope(qkv + (int64_t)h * d, d, (double)(pos + 1), w->rope_theta);", DRAFT),
    "draft_keys_not_rotated": ("for (int h = 0; h < hq + hk; ++h)\n            orc_rope(",
                               "for (int h = 0; h < hq; ++h)\n            orc_rope(", DRAFT),
    "draft_mlp_residual_from_x": ("            y[(int64_t)r * D + i] += x2[i];",
                                  "            y[(int64_t)r * D + i] += x[(int64_t)r * D + i];", DRAFT),
    "hsr_hidden_reads_first_half": ("o * 2 * D + D + i", "o * 2 * D + i", HSR),
    "argmax_ties_to_higher": ("if (isnan(z[best]) || z[x] > z[best])", "if (isnan(z[best]) || z[x] >= z[best])", GREEDY),
    "greedy_bonus_from_draft": ("out_tok[(int64_t)b * out_stride + n] = (int32_t)t_n;",
                                "out_tok[(int64_t)b * out_stride + n] = n > 0 ? draft[off_d + n - 1] : (int32_t)t_n;", GREEDY),
    "residual_without_clamp": ("w[x] = diff > 0.0 ? diff : 0.0;", "w[x] = fabs(diff);", SAMPLE),
    "ratio_inverted": ("r = exp(((double)zp[x] - orc_lse(zp, vocab)) - ((double)zq[x] - orc_lse(zq, vocab)));",
                       "r = exp(((double)zq[x] - orc_lse(zq, vocab)) - ((double)zp[x] - orc_lse(zp, vocab)));", SAMPLE),
    "bonus_from_first_row": ("const float *zp = tgt + (off_t + n) * vocab;\n        double lp",
                             "const float *zp = tgt + off_t * vocab;\n        double lp", SAMPLE),
    "draw_uses_first_uniform": ("(double)v[off_t + n]", "(double)v[off_t]", SAMPLE),
}


@pytest.fixture(scope="module")
def source():
    return open(obuild.SRC).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, source, tmp_path):
    old, new, pins = MUTANTS[name]
    assert source.count(old) == 1, f"mutation anchor for {name} must match exactly once"
    src = tmp_path / "sd_oracle.c"
    src.write_text(source.replace(old, new))
    (tmp_path / "sd_oracle.h").write_text(open(obuild.HDR).read())
    lib_path = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-fopenmp", "-o", str(lib_path),
                    str(src), "-lm"], check=True)
    real = oracle.lib()
    oracle._LIB = oracle.configure(ctypes.CDLL(str(lib_path)))
    failures = 0
    try:
        for pin in pins:
            try:
                pin()
            except (AssertionError, ValueError):
                failures += 1
    finally:
        oracle._LIB = real
    assert failures >= 1, f"no pin caught the planted mistake {name}"
