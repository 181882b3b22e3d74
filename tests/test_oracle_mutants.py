"""Mutation check of the oracle's pins: each plausible mistake, planted in a
copy of the oracle's C source on the CPU, must make at least one pin fail."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_q8_pins as q8pins
from tests import test_oracle_swiglu_pins as swpins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "q4_oracle.c")).read()

MUTANTS = {
    "nibble_halves_swapped": ("(blk[2 + j] & 0x0F) : (blk[2 + j - 16] >> 4)",
                              "(blk[2 + j] >> 4) : (blk[2 + j - 16] & 0x0F)"),
    "offset_7": ("(double)(q - 8) * d", "(double)(q - 7) * d"),
    "sign_dropped": ("(double)(q - 8) * d", "(double)(8 - q) * d"),
    "scale_big_endian": ("(uint16_t)(blk[0] | (blk[1] << 8))", "(uint16_t)(blk[1] | (blk[0] << 8))"),
    "block_stride_16": ("row + (k / 32) * 18", "row + (k / 32) * 16"),
    "code_index_off_by_one": ("blk[2 + j - 16] >> 4", "blk[2 + j - 15] >> 4"),
    "x_transposed": ("oracle_f16_to_f64(x[m * K + k])", "oracle_f16_to_f64(x[k * M + m])"),
    "f16_bias_16": ("ldexp((double)(1024 + f), e - 25)", "ldexp((double)(1024 + f), e - 26)"),
    "f16_subnormal_unit": ("ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    "acc_dropped_term": ("for (int64_t k = 0; k < K; ++k)\n                acc +=",
                         "for (int64_t k = 1; k < K; ++k)\n                acc +="),
    "repack_g_i_swapped": ("16 * (4 * g + c) + 4 * i + e", "16 * (4 * i + c) + 4 * g + e"),
    "repack_segment_stride": ("packed + 576 * (t * KB + b)", "packed + 512 * (t * KB + b)"),
    "repack_scale_slot": ("seg[512 + 8 * g + 2 * i + h]", "seg[512 + 8 * i + 2 * g + h]"),
    "repack_pad_code": ("(h < 2 ? 0x00 : 0x88)", "(h < 2 ? 0x00 : 0x00)"),
    "renorm_no_len": ("sqrt(s / (double)len)", "sqrt(s)"),
    "rne_ties_up": ("(frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))", "(frac >= 0.5)"),
}

# Planted in the Q8_0 part; caught by the Q8_0 pins.
Q8_MUTANTS = {
    "q8_codes_unsigned": ("(int)(int8_t)blk[2 + k % 32]", "(int)blk[2 + k % 32]"),
    "q8_block_stride_32": ("row + (k / 32) * 34", "row + (k / 32) * 32"),
    "q8_code_offset_1": ("blk[2 + k % 32]", "blk[1 + k % 32]"),
    "q8_repack_halves_swapped": ("seg[32 * (4 * g + c) + 8 * i + 4 + e] = blk[2 + 16 + 4 * c + e]",
                                 "seg[32 * (4 * g + c) + 8 * i + 4 + e] = blk[2 + 4 * c + e]"),
    "q8_repack_scale_slot": ("seg[1024 + 8 * g + 2 * i + h]", "seg[1024 + 8 * i + 2 * g + h]"),
    "q8_repack_segment_stride": ("packed + 1088 * (t * KB + b)", "packed + 1024 * (t * KB + b)"),
}

PIN_TESTS = [
    pins.test_f16_decoder_table,
    pins.test_f16_decoder_all_patterns_match_numpy,
    lambda: pins.test_f16_encoders("oracle"),
    pins.test_all_codes_eight_give_zero,
    pins.test_unit_vectors_pin_nibble_order_offset_and_scale,
    pins.test_single_nonzero_block,
    pins.test_linearity_in_scales,
    pins.test_brute_force_exact_rationals,
    pins.test_dense_matvec_equivalence_32x32_and_larger,
    pins.test_golden_hand_cases,
    lambda: pins.test_repack_round_trip_and_padding(40, 64),
    pins.test_renorm_invariants,
    pins.test_stack_chain_closed_form,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    assert old in SRC, f"mutation anchor for {name} no longer in the oracle"
    src = tmp_path / "mut.c"
    src.write_text(SRC.replace(old, new, 1))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           str(src), "-o", str(so), "-lm"])
    prev = oracle._swap_library(str(so))
    failed = []
    try:
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                failed.append(getattr(t, "__name__", "lambda"))
            except Exception:                      # a crash also counts as caught
                failed.append(getattr(t, "__name__", "lambda"))
    finally:
        oracle._restore_library(prev)
    assert failed, f"mutant {name} survived every pin"


Q8_PIN_TESTS = [
    q8pins.test_zero_codes_give_zero,
    q8pins.test_unit_vectors_pin_code_order_sign_and_scale,
    q8pins.test_scale_linearity_powers_of_two,
    q8pins.test_exact_rationals_brute_force,
    q8pins.test_dense_equivalence_synthetic_matrix,
    q8pins.test_repack_q8_round_trip_and_padding,
]


@pytest.mark.parametrize("name", sorted(Q8_MUTANTS))
def test_q8_mutant_is_caught(name, tmp_path):
    old, new = Q8_MUTANTS[name]
    assert old in SRC, f"mutation anchor for {name} no longer in the oracle"
    src = tmp_path / "mut.c"
    src.write_text(SRC.replace(old, new, 1))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           str(src), "-o", str(so), "-lm"])
    prev = oracle._swap_library(str(so))
    try:
        caught = 0
        for t in Q8_PIN_TESTS:
            try:
                t()
            except (AssertionError, ValueError, IndexError):
                caught += 1
        assert caught > 0, f"no Q8_0 pin catches mutant {name}"
    finally:
        oracle._restore_library(prev)


# Planted in the SiLU-gated input of the down GEMV; caught by its pins.
SWIGLU_MUTANTS = {
    "silu_exponent_sign": ("g / (1.0 + exp(-g)) * p", "g / (1.0 + exp(g)) * p"),
    "up_read_from_gate_half": ("oracle_f16_to_f64(v[K + k])", "oracle_f16_to_f64(v[k])"),
    "gate_without_silu": ("g / (1.0 + exp(-g)) * p", "g * p"),
    "f64_gemv_drops_last_column": ("for (int64_t k = 0; k < K; ++k)\n                acc += q4_0_weight(row, k) * x[m * K + k];",
                                   "for (int64_t k = 0; k < K - 1; ++k)\n                acc += q4_0_weight(row, k) * x[m * K + k];"),
}

SWIGLU_PIN_TESTS = [
    swpins.test_odd_part_of_silu_is_the_identity,
    swpins.test_taylor_series_at_zero_fixes_the_sign_of_the_exponent,
    swpins.test_limits,
    swpins.test_linear_in_the_up_half_and_gate_is_the_first_half,
    swpins.test_f64_gemv_matches_the_f16_gemv_on_f16_inputs,
    swpins.test_gated_gemv_dense_brute_force,
]


@pytest.mark.parametrize("name", sorted(SWIGLU_MUTANTS))
def test_swiglu_mutant_is_caught(name, tmp_path):
    old, new = SWIGLU_MUTANTS[name]
    assert old in SRC, f"mutation anchor for {name} no longer in the oracle"
    src = tmp_path / "mut.c"
    src.write_text(SRC.replace(old, new, 1))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           str(src), "-o", str(so), "-lm"])
    prev = oracle._swap_library(str(so))
    try:
        caught = 0
        for t in SWIGLU_PIN_TESTS:
            try:
                t()
            except (AssertionError, ValueError, IndexError):
                caught += 1
        assert caught > 0, f"no SiLU pin catches mutant {name}"
    finally:
        oracle._restore_library(prev)
