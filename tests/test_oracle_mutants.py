"""Plant plausible mistakes in copies of the CPU oracle and check that the
pins catch every one: a wrong scale offset, ties to odd, a lost sign of zero,
swapped nibbles, a reversed stochastic comparison, a transposed index, a wrong
Hadamard entry or normalisation, a wrong random stream, the tracker without
its absolute value, a reversed flag test, snapping to the old bin, a missing
reset, column groups built from X instead of Q_D(X), a wrong blocked scale
order, an overflow-aware bound taken inclusively. Mistakes are planted in
the oracle only, on the CPU; the real oracle source is never modified.
"""
import os
import subprocess

import pytest

import oracle as O
import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(O.__file__), "mxfp4_oracle.c")

# (name, original text, mutated text, pins that must fail)
MUTANTS = [
    ("Q-Ramping flag test inclusive", "flag[i] = d_q[i] > limit ? 1 : 0;",
     "flag[i] = d_q[i] >= limit ? 1 : 0;",
     ["test_qramp_flags_the_worked_oscillation_and_not_the_drift"]),
    ("Q-Ramping gathered update every iteration", "if (iter % k2 == k2 - 1) {",
     "if (1) {", ["test_qramp_flagged_weight_updates_every_k2th_iteration"]),
    ("Q-Ramping held updates dropped at the epoch start",
     "if (flag[i]) w[i] = (float)((double)w[i] + (double)acc[i]);", "",
     ["test_qramp_flagged_weight_updates_every_k2th_iteration"]),
    ("Q-Ramping window without the absolute value",
     "float moved_q = (float)fabs(qw[i] - qs[i]);",
     "float moved_q = (float)(qw[i] - qs[i]);",
     ["test_qramp_window_accumulates_like_the_tracker"]),
    ("overflow-aware bound inclusive", "ldexp(absmax, -e) > 6.0",
     "ldexp(absmax, -e) >= 6.0",
     ["test_oas_scale_is_the_smallest_non_saturating_exponent",
      "test_oas_moves_the_ocp_exponent_only_above_six"]),
    ("blocked lines and slots swapped", "16 * (tr % 32) + 4 * (tr / 32)",
     "4 * (tr % 32) + 16 * (tr / 32)",
     ["test_blocked_scales_line_by_line", "test_blocked_scales_is_a_padded_permutation"]),
    ("blocked tiles down the rows first", "(r / 128) * group_tiles + g / 4",
     "(g / 4) * row_tiles + r / 128", ["test_blocked_scales_line_by_line"]),
    ("scale offset", "int e = (E - 1) - 2;", "int e = (E - 1) - 1;",
     ["test_scale_exponent_exhaustive_bf16"]),
    ("ties to odd", "(dm == db && (m % 2) == 0)", "(dm == db && (m % 2) == 1)",
     ["test_rne_scalar_ties_and_saturation",
      "test_rne_exhaustive_bf16_times_every_scale_against_library"]),
    ("ties away from zero", "(dm == db && (m % 2) == 0)", "(dm == db)",
     ["test_hand_worked_groups"]),
    ("sign of zero lost", "(signbit(x) ? 8 : 0)", "(x < 0 ? 8 : 0)",
     ["test_sign_of_zero_codes", "test_hand_worked_groups"]),
    ("nibbles swapped", "  if (high)\n", "  if (!high)\n",
     ["test_rne_exhaustive_bf16_times_every_scale_against_library",
      "test_tiny_tensors_brute_force_layout"]),
    ("stochastic comparison reversed", "return (t < frac) ? lo + 1 : lo;",
     "return (t > frac) ? lo + 1 : lo;",
     ["test_sr_exhaustive_over_random_numbers_is_unbiased",
      "test_sr_end_to_end_unbiased_over_elements"]),
    ("stochastic step from the wrong bin",
     "double frac = (a - GRID[lo]) / (GRID[lo + 1] - GRID[lo]);",
     "double frac = (a - GRID[lo]) / 0.5;",
     ["test_sr_exhaustive_over_random_numbers_is_unbiased"]),
    ("column rng index transposed",
     "int64_t r = 32 * k + j;\n          idx[j] = (uint64_t)((row0 + r) * cols + c);",
     "int64_t r = 32 * k + j;\n          idx[j] = (uint64_t)(c * rows + r);",
     ["test_cols_sr_uses_input_row_major_index"]),
    ("column codes in row layout",
     "put_nibble(codes, c * (rows / 2) + r / 2, (int)(r & 1), cq[j]);",
     "put_nibble(codes, r * (cols / 2) + c / 2, (int)(c & 1), cq[j]);",
     ["test_tiny_tensors_brute_force_layout"]),
    ("random halves swapped", "return (i & 1) ? (h >> 16) : (h & 0xFFFFu);",
     "return (i & 1) ? (h & 0xFFFFu) : (h >> 16);",
     ["test_rand16_uniform_and_paired", "test_hash_frozen_known_answers"]),
    ("finalizer constant", "h *= 0x85EBCA6Bu;", "h *= 0x85EBCA6Du;",
     ["test_hash_finalizer_published_vectors"]),
    ("key stream constant", "stream * 0x9E3779B9u", "stream * 0x9E3779B1u",
     ["test_hash_frozen_known_answers"]),
    ("hadamard entry", "for (int b = j & k; b; b >>= 1)",
     "for (int b = j | k; b; b >>= 1)", ["test_rht_matches_scipy_hadamard"]),
    ("hadamard normalisation", "1.0 / sqrt(32.0)", "1.0 / 32.0",
     ["test_rht_matches_scipy_hadamard", "test_rht_orthonormal_properties"]),
    ("rht signs from the rounding stream", "orc_key(sign_seed, 1)",
     "orc_key(sign_seed, 0)", ["test_hash_frozen_known_answers"]),
    ("decode drops the sign", "return (code & 8) ? -v : v;", "return v;",
     ["test_decode_every_code_and_scale_against_library"]),
    ("double quant columns from X", "quantize_values(d, rows, cols, row0, AX_COLS",
     "quantize_values(xv, rows, cols, row0, AX_COLS",
     ["test_double_quant_structure"]),
    ("tracker without abs",
     "float dist_w = (float)fabs((double)w[i] - (double)w_snap[i]);",
     "float dist_w = (float)((double)w[i] - (double)w_snap[i]);",
     ["test_osc_accumulators_before_window_end"]),
    ("flag test reversed", "if (d_q[i] > limit) {", "if (d_q[i] < limit) {",
     ["test_osc_worked_example_from_the_page"]),
    ("snap to the old bin", "w[i] = (float)qw[i];", "w[i] = (float)qs[i];",
     ["test_osc_worked_example_from_the_page"]),
    ("no reset at window end", "      d_w[i] = 0.0f;\n", "",
     ["test_osc_accumulators_before_window_end"]),
    ("EMA weights swapped", "float keep = (float)((double)beta * (double)w_ema[i]);",
     "float keep = (float)((double)omb * (double)w_ema[i]);",
     ["test_qema_matches_the_geometric_closed_form"]),
    ("update sign bit", "(orc_counter_hash(k, gi) >> 31)",
     "(orc_counter_hash(k, gi) >> 30)",
     ["test_osc_synthetic_update_magnitude_and_signs"]),
]

PARAMS = {"test_tiny_tensors_brute_force_layout": [((32, 96), O.COLS),
                                                   ((64, 96), O.ROWS)],
          "test_qema_matches_the_geometric_closed_form": [(0.9, 200, 40)],
          "test_blocked_scales_line_by_line": [((300, 13),)]}


def _build(tmp_path, name, src_text):
    c = tmp_path / (name.replace(" ", "_") + ".c")
    so = tmp_path / (name.replace(" ", "_") + ".so")
    c.write_text(src_text)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-fPIC",
                    "-shared", "-o", str(so), str(c), "-lm"], check=True)
    return O.Oracle(str(so))


def _run_pin(lib, pin):
    """Run pin against lib; True if it passed."""
    saved = P.O
    P.O = lib
    try:
        fn = getattr(P, pin)
        for args in PARAMS.get(pin, [()]):
            fn(*args)
        return True
    except AssertionError:
        return False
    finally:
        P.O = saved


def test_unmutated_copy_passes_every_selected_pin(tmp_path):
    lib = _build(tmp_path, "clean", open(SRC).read())
    for pin in sorted({p for m in MUTANTS for p in m[3]}):
        assert _run_pin(lib, pin), pin


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, mutant):
    name, old, new, pins = mutant
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site not unique: %s" % name
    lib = _build(tmp_path, name, src.replace(old, new))
    caught = [p for p in pins if not _run_pin(lib, p)]
    assert caught, "no pin caught the mutant '%s'" % name
