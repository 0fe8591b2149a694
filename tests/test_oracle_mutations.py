"""The pins catch plausible mistakes in the oracle.

Each mutant is a copy of oracle/swa_oracle.c with one planted mistake (an
off-by-one window, a flipped causal bound, a dropped scale or denominator, a
transposed operand, a wrong head map, a wrong ring or chunk index, a swapped
tile class, a gradient without its D term, ...), compiled into a temporary directory.  The pins of
tests/test_oracle_pins.py run against the mutant through oracle.use_library;
every mutant must make at least one of them fail.  The committed oracle is
never modified.
"""

import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "swa_oracle.c")

MUTANTS = {
    "window_off_by_one": ("(j >= i - W + 1)", "(j >= i - W)"),
    "sees_one_future_key": ("return (j <= i) &&", "return (j <= i + 1) &&"),
    "scale_dropped": ("s *= scale;", "s *= 1.0;"),
    "key_value_transposed": ("bf16_value(qrow[c]) * bf16_value(krows[t][c])",
                             "bf16_value(qrow[c]) * bf16_value(vrows[t][c])"),
    "denominator_dropped": ("double w = scores[t] / denom;", "double w = scores[t];"),
    "value_dim_shifted": ("out[c] += w * bf16_value(vrows[t][c]);",
                          "out[c] += w * bf16_value(vrows[t][(c + 1) % d]);"),
    "lse_without_max": ("*lse = smax + log(denom);", "*lse = log(denom);"),
    "gqa_map_modulo": ("return h / (H / Hkv);", "return h % Hkv;"),
    "ring_start_step": ("start = (start + 1) % W;", "start = (start + 2) % W;"),
    "chunk_row_shift": ("int64_t row = j - q_start[b];\n",
                        "int64_t row = (j - q_start[b] + 1) % Tq;\n"),
    "decode_ring_one_short": ("orc_ring_positions(pos[b] + 1, W, maps + b * W);",
                              "orc_ring_positions(pos[b], W, maps + b * W);"),
    "dense_mask_diff_gt": ("(diff < 0 || diff >= W)", "(diff < 0 || diff > W)"),
    "tile_full_partial_swapped": ("int8_t cls = n_ok == 0 ? 0 : (n_ok == n_in ? 1 : 2);",
                                  "int8_t cls = n_ok == 0 ? 0 : (n_ok == n_in ? 2 : 1);"),
    "tile_rows_clipped_short": (
        "int64_t r_end = r_begin + tile_q < n_q ? r_begin + tile_q : n_q;",
        "int64_t r_end = r_begin + tile_q - 1 < n_q ? r_begin + tile_q - 1 : n_q;"),
    "count_pairs_strict": ("n += allowed(i, j, W);", "n += allowed(i, j, W) && j < i;"),
    "sink_count_inclusive": ("(j >= i - W + 1 || j < S)", "(j >= i - W + 1 || j <= S)"),
    "sink_pairs_ignore_sinks": ("n += allowed_sink(i, j, W, S);", "n += allowed(i, j, W);"),
    "varlen_sequence_base_dropped": ("kr[n] = k + ((first + j) * Hkv + kh) * d;",
                                     "kr[n] = k + (j * Hkv + kh) * d;"),
    "varlen_boundary_token_misassigned": (
        "while (s + 1 < n_seq && cu_seqlens[s + 1] <= t) ++s;",
        "while (s + 1 < n_seq && cu_seqlens[s + 1] < t) ++s;"),
    "decode_sink_row_fixed": ("kr[n] = sink_k + ((b * Hkv + kh) * S + j) * d;",
                              "kr[n] = sink_k + ((b * Hkv + kh) * S + 0) * d;"),
    "decode_sink_window_edge": ("if (j >= p - W + 1) {", "if (j > p - W + 1) {"),
    "backward_delta_dropped": ("double ds = p[j - lo] * (dp[j - lo] - Di);",
                               "double ds = p[j - lo] * dp[j - lo];"),
    "backward_dk_unscaled": ("dkj[c] += scale * ds * qi[c];", "dkj[c] += ds * qi[c];"),
    "backward_dv_from_q": ("dvj[c] += p[j - lo] * gi[c];", "dvj[c] += p[j - lo] * qi[c];"),
    "backward_dq_from_q": ("dqi[c] += scale * ds * kj[c];", "dqi[c] += scale * ds * qi[c];"),
    "varlen_backward_delta_dropped": ("double ds = p[t] * (dp[t] - Di);",
                                      "double ds = p[t] * dp[t];"),
    "varlen_backward_dk_unscaled": ("dk[row * d + c] += scale * ds * qi[c];",
                                    "dk[row * d + c] += ds * qi[c];"),
    "varlen_backward_dv_from_q": ("dv[row * d + c] += p[t] * gi[c];",
                                  "dv[row * d + c] += p[t] * qi[c];"),
    "varlen_backward_sequence_base_dropped": ("int64_t row = (first + idx[t]) * Hkv + kh;",
                                              "int64_t row = idx[t] * Hkv + kh;"),
    "varlen_f64_sinks_ignored": ("if (allowed_sink(i, j, W, S)) idx[n++] = j;",
                                 "if (allowed(i, j, W)) idx[n++] = j;"),
}


def _pin_suite(golden_dir):
    """Every pin as a zero-argument call (parametrised pins at representative values)."""
    return [
        lambda: pins.test_valid_pairs_worked_example(golden_dir),
        lambda: pins.test_valid_pairs_closed_form(100, 7),
        lambda: pins.test_visible_sets_worked_example(golden_dir),
        lambda: pins.test_visible_sets_chapter10(golden_dir),
        lambda: pins.test_zero_scores_last_query(golden_dir),
        lambda: pins.test_tile_coverage_worked_example(golden_dir),
        lambda: pins.test_tile_classes_consistent_with_pairs(200, 37, 64, 32),
        lambda: pins.test_tile_classes_ring_mode_counts(),
        lambda: pins.test_full_window_equals_causal_sdpa(2, 4, 2, 37, 16),
        lambda: pins.test_window_one_returns_own_value(),
        lambda: pins.test_loop_oracle_equals_dense_mask(7),
        lambda: pins.test_ring_positions_slot_is_pos_mod_w(8),
        lambda: pins.test_ring_update_keeps_latest_positions(),
        lambda: pins.test_chunk_union_chapter10(golden_dir),
        lambda: pins.test_full_equals_chunked_chapter10(golden_dir),
        lambda: pins.test_full_equals_chunked_general(16, [(0, 5), (5, 40), (40, 41), (41, 90)]),
        lambda: pins.test_decode_equals_prefill_row(16, 50),
        lambda: pins.test_lse_matches_definition(),
        lambda: pins.test_sink_pairs_closed_form(100, 7, 4),
        lambda: pins.test_sink_pairs_special_cases(),
        lambda: pins.test_varlen_visible_sets([8, 5, 1, 12], 3, 4),
        lambda: pins.test_varlen_first_token_returns_own_value(),
        lambda: pins.test_varlen_single_sequence_equals_linear_forward(),
        lambda: pins.test_varlen_reduces_to_causal_sdpa(1000, 0),
        lambda: pins.test_varlen_no_cross_talk(),
        lambda: pins.test_sink_tokens_influence_and_middle_tokens_do_not(),
        lambda: pins.test_decode_sink_equals_prefill_row(8, 4, 12),
        lambda: pins.test_decode_sink_equals_prefill_row(16, 4, 50),
        lambda: pins.test_chunked_with_sinks_equals_full(16, 4, [(0, 5), (5, 40), (40, 41),
                                                                  (41, 90)]),
        lambda: pins.test_forward_f64_equals_forward(),
        lambda: pins.test_backward_finite_differences(3),
        lambda: pins.test_backward_full_window_equals_torch_autograd(1, 4, 2, 37, 16),
        lambda: pins.test_backward_window_one(),
        lambda: pins.test_varlen_backward_finite_differences(3, 2),
        lambda: pins.test_varlen_backward_equals_dense_mask_autograd([7, 3, 12], 4, 2),
        lambda: pins.test_varlen_backward_single_sequence_equals_linear(),
        lambda: pins.test_varlen_backward_no_cross_talk(),
        lambda: pins.test_varlen_backward_window_one(),
    ]


def test_committed_oracle_passes_the_suite(golden_dir):
    for pin in _pin_suite(golden_dir):
        pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, golden_dir, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib),
                    str(src), "-lm"], check=True)
    failed = []
    with oracle.use_library(str(lib)):
        for i, pin in enumerate(_pin_suite(golden_dir)):
            try:
                pin()
            except (AssertionError, ValueError):
                failed.append(i)
    assert failed, f"no pin catches the mutant {name}"
