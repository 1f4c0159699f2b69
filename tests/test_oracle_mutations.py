"""Planted mistakes in the oracle must fail at least one pin.

Each case copies ``oracle/tq_oracle.cpp`` to a temporary directory, plants one
plausible mistake (a wrong sign, a dropped term, a wrong index, a transposed
operand), compiles it, and runs the fast pins from ``test_oracle_pins`` against
the mutated library. The committed oracle is never modified.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle.build import CXXFLAGS, SRC
from tests import test_oracle_pins as pins

MUTATIONS = {
    "fwht_difference_sign": ("u[i + h] = a - b;", "u[i + h] = b - a;"),
    "norm_const_1_over_D": ("return (float)(1.0 / std::sqrt((double)D));", "return (float)(1.0 / (double)D);"),
    "scale_divisor_8": ("const float sigma32 = a / 7.0f;", "const float sigma32 = a / 8.0f;"),
    "truncate_not_round": ("float c = std::nearbyint(r);", "float c = std::trunc(r);"),
    "nibbles_swapped": ("bytes[j] = (uint8_t)(lo | (hi << 4));", "bytes[j] = (uint8_t)(hi | (lo << 4));"),
    "forward_sign_dropped": ("for (int i = 0; i < D; ++i) u[i] = s[i] * x[i];", "for (int i = 0; i < D; ++i) u[i] = x[i];"),
    "inverse_sign_dropped": ("for (int i = 0; i < D; ++i) x[i] = s[i] * (u[i] * c);",
                             "for (int i = 0; i < D; ++i) x[i] = u[i] * c;"),
    "gqa_map_modulo": ("const int kv = hq / G;", "const int kv = hq % n_kv;"),
    "softmax_scale_dropped": ("z[t] = (double)sm_scale * dot;", "z[t] = dot;"),
    "softmax_not_normalised": ("const double w = z[t] / l;", "const double w = z[t];"),
    "k_used_for_v": ("dequantize_rotated(v_codes + row * cb, v_scales + row * sb, D, yv.data());",
                     "dequantize_rotated(k_codes + row * cb, k_scales + row * sb, D, yv.data());"),
    "f16_ties_away": ("if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;", "if (rem >= 0x1000u) h += 1u;"),
    "f16_exponent_bias": ("uint32_t h = ((uint32_t)(e + 15) << 10) | (frac >> 13);",
                          "uint32_t h = ((uint32_t)(e + 14) << 10) | (frac >> 13);"),
}


def quick_f16_pin(orc):
    """A fast sample of the exhaustive binary16 pin, with forced round-to-even ties."""
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    bits[: 1 << 12] = (bits[: 1 << 12] & ~np.uint32(0x1FFF)) | np.uint32(0x1000)  # exact ties
    x = bits.view(np.float32)
    got = orc.f32_to_f16_bits(x)
    ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    keep = ~np.isnan(x)
    assert np.array_equal(got[keep], ref[keep])


def fast_pins(orc):
    yield lambda: pins.test_fwht_equals_sylvester_matrix(orc, 128)
    yield lambda: pins.test_srht_orthonormal_inverse_parseval(orc, 128)
    yield lambda: pins.test_closed_form_unit_vector(orc, 64)
    yield lambda: pins.test_closed_form_hadamard_column(orc, 128)
    yield lambda: pins.test_quantiser_against_brute_force(orc, 128)
    yield lambda: pins.test_pack_unpack_identity(orc)
    yield lambda: pins.test_attention_equals_fp64_original_domain(orc, 128, 8, 2, 33)
    yield lambda: pins.test_attention_special_cases(orc)
    yield lambda: pins.test_f16_to_f32_exhaustive(orc)
    yield lambda: quick_f16_pin(orc)


def failing_pins(orc):
    failed = 0
    for check in fast_pins(orc):
        try:
            check()
        except AssertionError:
            failed += 1
    return failed


def test_fast_pins_pass_on_committed_oracle(orc):
    assert failing_pins(orc) == 0


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "tq_oracle_mut.cpp"
    mutated.write_text(src.replace(before, after))
    lib_path = tmp_path / f"libtq_oracle_{name}.so"
    subprocess.run(["g++", *CXXFLAGS, "-o", str(lib_path), str(mutated)], check=True)
    lib = oracle.bind(ctypes.CDLL(os.fspath(lib_path)))
    monkeypatch.setattr(oracle, "_lib", lib)
    assert failing_pins(oracle) >= 1, f"no pin caught the planted mistake {name}"


# Planted mistakes in the asymmetric (binary16 K) path, checked by its own pins.
KF16_MUTATIONS = {
    "kf16_k_index_reversed": ("    dst[i] = hbits;", "    dst[D - 1 - i] = hbits;"),
    "kf16_q_rotated": ("std::memcpy(qr.data(), q + ((int64_t)b * n_q + hq) * D, sizeof(float) * D);",
                       "srht_forward_vec(q + ((int64_t)b * n_q + hq) * D, s, D, qr.data());"),
    "kf16_k_halved": ("for (int i = 0; i < D; ++i) yk[i] = f16_to_f32(k_f16[row * D + i]);",
                      "for (int i = 0; i < D; ++i) yk[i] = 0.5f * f16_to_f32(k_f16[row * D + i]);"),
}


def kf16_pins(orc):
    yield lambda: pins.test_kf16_append_stores_numpy_binary16_and_the_symmetric_v(orc, 128)
    yield lambda: pins.test_kf16_attention_equals_fp64_original_domain(orc, 128, 16, 2, 33)
    yield lambda: pins.test_kf16_attention_special_cases(orc)


def failing_kf16_pins(orc):
    failed = 0
    for check in kf16_pins(orc):
        try:
            check()
        except AssertionError:
            failed += 1
    return failed


def test_kf16_pins_pass_on_committed_oracle(orc):
    assert failing_kf16_pins(orc) == 0


@pytest.mark.parametrize("name", sorted(KF16_MUTATIONS))
def test_planted_kf16_mistake_is_caught(name, tmp_path, monkeypatch):
    before, after = KF16_MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "tq_oracle_mut.cpp"
    mutated.write_text(src.replace(before, after))
    lib_path = tmp_path / f"libtq_oracle_{name}.so"
    subprocess.run(["g++", *CXXFLAGS, "-o", str(lib_path), str(mutated)], check=True)
    lib = oracle.bind(ctypes.CDLL(os.fspath(lib_path)))
    monkeypatch.setattr(oracle, "_lib", lib)
    assert failing_kf16_pins(oracle) >= 1, f"no pin caught the planted mistake {name}"


DELEGATED_MUTATIONS = {
    "deleg_cold_length_floor": ("return (len - W + F - 1) / F * F;", "return (len - W) / F * F;"),
    "deleg_fold_reads_next_slot": ("const uint16_t* hot = v_tail + (((int64_t)b * W + T % W) * n_kv + h) * D;",
                                   "const uint16_t* hot = v_tail + (((int64_t)b * W + (T + 1) % W) * n_kv + h) * D;"),
    "deleg_tail_written_one_slot_late": ("uint16_t* hot = v_tail + (((int64_t)b * W + P % W) * n_kv + h) * D;",
                                         "uint16_t* hot = v_tail + (((int64_t)b * W + (P + 1) % W) * n_kv + h) * D;"),
    "deleg_hot_v_not_rotated": ("srht_forward_vec(xv.data(), s, D, yv.data());",
                                "std::memcpy(yv.data(), xv.data(), sizeof(float) * D);"),
    "deleg_tail_holds_k": ("hot[i] = vb;", "hot[i] = kb;"),
    "deleg_boundary_token_read_cold": ("if (t < n_cold) {", "if (t <= n_cold) {"),
}


def delegated_pins(orc):
    yield lambda: pins.test_delegated_cold_length_worked_values_and_invariants(orc)
    yield lambda: pins.test_delegated_append_holds_binary16_tail_and_encoded_body(orc, 128, 8, 4, 13)
    yield lambda: pins.test_delegated_append_is_chunking_invariant(orc)
    yield lambda: pins.test_delegated_attention_equals_fp64(orc, 128, 8, 1, 16, 8, 50)
    yield lambda: pins.test_delegated_all_hot_is_binary16_attention_of_the_inputs(orc)
    yield lambda: pins.test_delegated_special_cases(orc)


def failing_delegated_pins(orc):
    failed = 0
    for check in delegated_pins(orc):
        try:
            check()
        except AssertionError:
            failed += 1
    return failed


def test_delegated_pins_pass_on_committed_oracle(orc):
    assert failing_delegated_pins(orc) == 0


@pytest.mark.parametrize("name", sorted(DELEGATED_MUTATIONS))
def test_planted_delegated_mistake_is_caught(name, tmp_path, monkeypatch):
    before, after = DELEGATED_MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "tq_oracle_mut.cpp"
    mutated.write_text(src.replace(before, after))
    lib_path = tmp_path / f"libtq_oracle_{name}.so"
    subprocess.run(["g++", *CXXFLAGS, "-o", str(lib_path), str(mutated)], check=True)
    lib = oracle.bind(ctypes.CDLL(os.fspath(lib_path)))
    monkeypatch.setattr(oracle, "_lib", lib)
    assert failing_delegated_pins(oracle) >= 1, f"no pin caught the planted mistake {name}"


EXT_MUTATIONS = {
    "lambda_divides_instead": ("      for (int i = 0; i < D; ++i) y[i] = y[i] * lambda[i];",
                               "      for (int i = 0; i < D; ++i) y[i] = y[i] / lambda[i];"),
    "lambda_before_transform": ("    srht_forward_vec(x + v * D, s, D, y.data());\n    if (lambda)\n      for (int i = 0; i < D; ++i) y[i] = y[i] * lambda[i];",
                                "    std::vector<float> xl(x + v * D, x + v * D + D);\n    if (lambda)\n      for (int i = 0; i < D; ++i) xl[i] = xl[i] * lambda[i];\n    srht_forward_vec(xl.data(), s, D, y.data());"),
    "lambda_k_not_undone": ("dot += (double)qr[i] * ((double)yk[i] / (double)lambda_k[i]);",
                            "dot += (double)qr[i] * (double)yk[i];"),
    "lambda_v_not_undone": ("acc[i] += w * ((double)yv[i] / (double)lambda_v[i]);", "acc[i] += w * (double)yv[i];"),
    "sparse_normalised_weight": ("const bool dropped = tau > 0.0 && t < n_cold && z[t] < tau;",
                                 "const bool dropped = tau > 0.0 && t < n_cold && z[t] / l < tau;"),
    "sparse_drops_the_sum_too": ("        z[t] = std::exp(z[t] - m);\n        l += z[t];",
                                 "        z[t] = std::exp(z[t] - m);\n        l += (tau > 0.0 && z[t] < tau) ? 0.0 : z[t];"),
}


def ext_pins(orc):
    yield lambda: pins.test_lambda_sits_between_the_transform_and_the_abs_max(orc)
    yield lambda: pins.test_lambda_powers_of_two_per_group_keep_codes_and_shift_scales(orc)
    yield lambda: pins.test_lambda_attention_equals_fp64(orc, 128, 8, 2, 40)
    yield lambda: pins.test_sparse_v_zero_threshold_is_exact_and_the_drop_rule(orc)


def failing_ext_pins(orc):
    failed = 0
    for check in ext_pins(orc):
        try:
            check()
        except AssertionError:
            failed += 1
    return failed


def test_ext_pins_pass_on_committed_oracle(orc):
    assert failing_ext_pins(orc) == 0


@pytest.mark.parametrize("name", sorted(EXT_MUTATIONS))
def test_planted_lambda_or_sparse_mistake_is_caught(name, tmp_path, monkeypatch):
    before, after = EXT_MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "tq_oracle_mut.cpp"
    mutated.write_text(src.replace(before, after))
    lib_path = tmp_path / f"libtq_oracle_{name}.so"
    subprocess.run(["g++", *CXXFLAGS, "-o", str(lib_path), str(mutated)], check=True)
    lib = oracle.bind(ctypes.CDLL(os.fspath(lib_path)))
    monkeypatch.setattr(oracle, "_lib", lib)
    assert failing_ext_pins(oracle) >= 1, f"no pin caught the planted mistake {name}"


PAGED_MUTATIONS = {
    "paged_append_row_shifted": ("const int64_t prow = (int64_t)pg * P + pos % P;",
                                 "const int64_t prow = (int64_t)pg * P + (pos + 1) % P;"),
    "paged_gather_row_shifted": ("const int64_t src = ((int64_t)pg * P + t % P) * n_kv + h;",
                                 "const int64_t src = ((int64_t)pg * P + (t + 1) % P) * n_kv + h;"),
    "paged_page_index_off_by_one": ("const int pg = table[(int64_t)b * max_pages + pos / P];",
                                    "const int pg = table[(int64_t)b * max_pages + (pos + 1) / P];"),
}


def failing_paged_pins(orc):
    failed = 0
    for check in (lambda: pins.test_paged_cache_is_the_contiguous_cache_with_rows_moved(orc, False),
                  lambda: pins.test_paged_cache_is_the_contiguous_cache_with_rows_moved(orc, True),
                  lambda: pins.test_paged_unmapped_page_is_skipped_with_status(orc)):
        try:
            check()
        except AssertionError:
            failed += 1
    return failed


def test_paged_pins_pass_on_committed_oracle(orc):
    assert failing_paged_pins(orc) == 0


@pytest.mark.parametrize("name", sorted(PAGED_MUTATIONS))
def test_planted_paged_mistake_is_caught(name, tmp_path, monkeypatch):
    before, after = PAGED_MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "tq_oracle_mut.cpp"
    mutated.write_text(src.replace(before, after))
    lib_path = tmp_path / f"libtq_oracle_{name}.so"
    subprocess.run(["g++", *CXXFLAGS, "-o", str(lib_path), str(mutated)], check=True)
    lib = oracle.bind(ctypes.CDLL(os.fspath(lib_path)))
    monkeypatch.setattr(oracle, "_lib", lib)
    assert failing_paged_pins(oracle) >= 1, f"no pin caught the planted mistake {name}"
