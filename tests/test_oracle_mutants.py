"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it as a separate module, and runs the pins of
test_oracle_pins.py against it: at least one pin must fail.  An unmodified copy
must pass them all, which shows the harness itself is sound.
"""
import importlib.util
import os
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_DIR = os.path.join(os.path.dirname(HERE), "oracle")


def _load_pins():
    spec = importlib.util.spec_from_file_location("oracle_pins_for_mutants",
                                                  os.path.join(HERE, "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PINS = _load_pins()

# (pin, keyword arguments): one representative parameter set per pin
PIN_CALLS = [
    ("test_hadamard_sylvester_recursion_and_scipy", {}),
    ("test_rotation_is_orthonormal_hadamard_times_signs", {"d": 64}),
    ("test_rotation_rejects_bad_signs", {}),
    ("test_lloyd_max_one_bit_closed_form", {}),
    ("test_lloyd_max_conditions_by_quadrature", {"b": 3}),
    ("test_lloyd_max_matches_classical_table_and_is_a_minimum", {"b": 4}),
    ("test_codebook_scaling_symmetry_and_boundaries", {"d": 128, "b": 3}),
    ("test_codebook_is_data_independent", {}),
    ("test_packing_hand_worked_examples", {}),
    ("test_pack_roundtrip_and_bit_positions", {"d": 16, "b": 3}),
    ("test_rotated_unit_keys_have_unit_norm_and_variance_one_over_d", {}),
    ("test_basis_vector_closed_form", {"b": 2}),
    ("test_zero_key", {}),
    ("test_brute_force_nearest_codeword_d8", {"b": 2}),
    ("test_quantization_mse_matches_lloyd_max", {"b": 4}),
    ("test_margins_are_distances_to_decision_points", {}),
    ("test_lut_scores_equal_dequantized_dot", {"d": 64, "b": 3, "group": 2}),
    ("test_scores_brute_force_d8", {}),
    ("test_attention_of_equal_scores_is_the_mean_value_row", {}),
    ("test_attention_single_key_returns_its_value_row", {}),
    ("test_attention_brute_force_on_dequantized_keys", {}),
    ("test_attention_is_linear_in_values_and_shift_free_in_scores", {}),
    ("test_sign_errors_brute_force_d8", {"b": 2}),
    ("test_sign_errors_planted_pattern_closed_form", {"b": 4}),
    ("test_sign_errors_symmetries_and_scaling", {}),
    ("test_sign_errors_are_means_over_samples_queries_and_keys", {}),
    ("test_sign_errors_match_lloyd_max_distortion", {"b": 3}),
    ("test_select_signs_worst_head_and_lowest_index", {}),
    ("test_block_rotation_follows_hamilton_rules", {}),
    ("test_block_rotation_is_orthonormal_and_block_diagonal", {}),
    ("test_block_rotation_isoclinic_and_conjugation_closed_forms", {}),
    ("test_block_quantize_and_scores_brute_force_d8", {"b": 2}),
    ("test_block_lut_scores_equal_dequantized_dot", {"d": 128, "b": 4}),
    ("test_block_quantization_mse_matches_lloyd_max_on_isotropic_keys", {"b": 4}),
]

# name -> (text in oracle.c, replacement): one plausible mistake each
MUTANTS = {
    "sign_flip_dropped": (
        "R[(size_t)i * d + j] *= (double)signs[j] * inv_sqrt_d;",
        "R[(size_t)i * d + j] *= inv_sqrt_d;"),
    "signs_applied_to_rows": (
        "R[(size_t)i * d + j] *= (double)signs[j] * inv_sqrt_d;",
        "R[(size_t)i * d + j] *= (double)signs[i] * inv_sqrt_d;"),
    "rotation_not_normalised": (
        "R[(size_t)i * d + j] *= (double)signs[j] * inv_sqrt_d;",
        "R[(size_t)i * d + j] *= (double)signs[j];"),
    "codebook_scaled_by_1_over_d": (
        "const double sigma = 1.0 / sqrt((double)d);",
        "const double sigma = 1.0 / (double)d;"),
    "centroid_rule_replaced_by_cell_midpoint": (
        "next[i] = std_normal_conditional_mean(lo, hi);",
        "next[i] = (i == 0) ? hi - 1.0 : (i == L - 1) ? lo + 1.0 : 0.5 * (lo + hi);"),
    "ties_to_upper_index": (
        "if (dist < best_dist) {",
        "if (dist <= best_dist) {"),
    "msb_first_packing": (
        "if ((codes[j] >> i) & 1) row[bit / 8] |= (uint8_t)(1u << (bit % 8));",
        "if ((codes[j] >> i) & 1) row[bit / 8] |= (uint8_t)(1u << (7 - bit % 8));"),
    "temperature_dropped": (
        "out[t] = (double)norms[(int64_t)h * n + t] * s * inv_sqrt_d;",
        "out[t] = (double)norms[(int64_t)h * n + t] * s;"),
    "query_reads_wrong_kv_head": (
        "unpack_row(packed + ((int64_t)h * n + t) * P, d, b, codes);\n                double s = 0.0;",
        "unpack_row(packed + ((int64_t)((h * group + g) % heads) * n + t) * P, d, b, codes);\n"
        "                double s = 0.0;"),
    "squared_norm_stored": (
        "const float norm = (float)sqrt(ss);",
        "const float norm = (float)ss;"),
    "block_right_factor_not_conjugated": (
        "const double qRc[4] = {qR[0], -qR[1], -qR[2], -qR[3]};",
        "const double qRc[4] = {qR[0], qR[1], qR[2], qR[3]};"),
    "hamilton_cross_term_sign": (
        "out[1] = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];",
        "out[1] = a[0] * b[1] + a[1] * b[0] - a[2] * b[3] + a[3] * b[2];"),
    "block_matrix_transposed": (
        "for (int r = 0; r < 4; ++r) R[(size_t)(4 * m + r) * d + 4 * m + c] = y[r];",
        "for (int r = 0; r < 4; ++r) R[(size_t)(4 * m + c) * d + 4 * m + r] = y[r];"),
    "boundary_at_lower_centroid": (
        "boundaries[i] = (float)(0.5 * ((double)centroids[i] + (double)centroids[i + 1]));",
        "boundaries[i] = centroids[i];"),
}

# mistakes in the Python half of the oracle (__init__.py): name -> (text, replacement)
PY_MUTANTS = {
    "attention_reads_wrong_value_head": (
        "out[h * group:(h + 1) * group] = p[h * group:(h + 1) * group] @ V[h]",
        "out[h * group:(h + 1) * group] = p[h * group:(h + 1) * group] @ V[(h + 1) % heads]"),
    "softmax_not_normalised": (
        "    p /= p.sum(axis=1, keepdims=True)\n",
        ""),
    "exact_logit_without_temperature": (
        "exact = q[s, rows] @ K[s, h].T / np.sqrt(d)",
        "exact = q[s, rows] @ K[s, h].T"),
    "sign_error_mean_over_keys_only": (
        "return sq / (S * group * n)",
        "return sq / n"),
    "queries_read_with_first_candidate": (
        "norms.reshape(heads, n), group, b, cand[c])",
        "norms.reshape(heads, n), group, b, cand[0])"),
    "selection_by_mean_over_heads": (
        "worst = np.asarray(errors, dtype=np.float64).max(axis=1)",
        "worst = np.asarray(errors, dtype=np.float64).mean(axis=1)"),
}

# the MSB-first mutant changes packing on both sides, as a consistent mistake would
UNPACK_MSB = ("v |= (unsigned)((row[bit / 8] >> (bit % 8)) & 1) << i;",
              "v |= (unsigned)((row[bit / 8] >> (7 - bit % 8)) & 1) << i;")


def _build_copy(tmp_path, name, edits, py_edits=()):
    pkg = tmp_path / f"oracle_{name}"
    pkg.mkdir()
    src = open(os.path.join(ORACLE_DIR, "oracle.c")).read()
    for old, new in edits:
        assert src.count(old) == 1, f"{name}: edit target not found once: {old}"
        src = src.replace(old, new)
    (pkg / "oracle.c").write_text(src)
    py = open(os.path.join(ORACLE_DIR, "__init__.py")).read()
    for old, new in py_edits:
        assert py.count(old) == 1, f"{name}: edit target not found once: {old}"
        py = py.replace(old, new)
    (pkg / "__init__.py").write_text(py)
    modname = f"oracle_copy_{name}"
    spec = importlib.util.spec_from_file_location(modname, pkg / "__init__.py",
                                                  submodule_search_locations=[str(pkg)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[modname] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _failing_pins(monkeypatch, mod):
    monkeypatch.setattr(PINS, "oracle", mod)
    failed = []
    for pin, kw in PIN_CALLS:
        try:
            getattr(PINS, pin)(**kw)
        except Exception as e:          # an assertion, or the oracle rejecting its inputs
            failed.append((pin, type(e).__name__))
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path, monkeypatch):
    mod = _build_copy(tmp_path, "unmodified", [])
    assert _failing_pins(monkeypatch, mod) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(tmp_path, monkeypatch, name):
    edits = [MUTANTS[name]] + ([UNPACK_MSB] if name == "msb_first_packing" else [])
    mod = _build_copy(tmp_path, name, edits)
    failed = _failing_pins(monkeypatch, mod)
    assert failed, f"no pin catches the planted mistake {name}"


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_planted_mistake_in_the_python_half_fails_a_pin(tmp_path, monkeypatch, name):
    mod = _build_copy(tmp_path, name, [], [PY_MUTANTS[name]])
    failed = _failing_pins(monkeypatch, mod)
    assert failed, f"no pin catches the planted mistake {name}"
