"""The CPU oracle against what the pages and mathematics fix (runs without a GPU)."""
import pytest

import oracle_pins as P


def test_fp16_golden():
    P.pin_fp16_golden()


def test_fp16_rounding_vs_numpy():
    P.pin_fp16_vs_numpy()


def test_fp16_decode_all_bit_patterns():
    P.pin_fp16_decode_all()


def test_hadamard_is_blockdiag_sylvester():
    P.pin_hadamard_matrix()


def test_hadamard_golden():
    P.pin_hadamard_golden()


def test_hadamard_exact_on_integers():
    P.pin_hadamard_integer_exact()


def test_quantiser_golden():
    P.pin_quant_golden()


def test_int4_quantiser_bounds_and_independent_requant():
    P.pin_quant_int4_bounds()


def test_int4_constant_vector_exact():
    P.pin_quant_int4_constant()


def test_int8_quantiser_bounds():
    P.pin_quant_int8_bounds()


def test_storage_bits_per_element():
    P.pin_storage_bits()


def test_layout_is_a_bijection():
    P.pin_layout_bijection()


@pytest.mark.parametrize("step_by_step", [False, True])
def test_sink_and_ring_routing(step_by_step):
    P.pin_routing(step_by_step)


def test_brute_force_tiny():
    P.pin_brute_force()


def test_append_matches_independent_requant():
    P.pin_append_vs_numpy_requant()


def test_regional_merge_equals_single_softmax():
    P.pin_regional_equals_single()


def test_rotation_invariance():
    P.pin_rotation_invariance()


def test_signed_rotation_exact():
    P.pin_signed_rotation_exact()


def test_value_rotation_invariance():
    P.pin_value_rotation_invariance()


def test_special_cases():
    P.pin_special_cases()


def test_quantiser_range_overflow():
    P.pin_quant_range()


def test_append_reports_range_overflow():
    P.pin_append_range_flag()


def test_bf16_rounding():
    P.pin_bf16_rounding()


def test_bf16_value_layout_is_a_bijection():
    P.pin_layout_bijection_bf16_values()


def test_bf16_values_stored_exactly():
    P.pin_bf16_values_exact()
