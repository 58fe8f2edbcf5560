"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a dropped
term, a wrong index or sign, a transposed operand, a wrong rounding or
order), compiles it, points the oracle module at the mutant and runs the pin
battery of tests/test_oracle_*.py on it: at least one pin must fail.
Mistakes are planted only in the oracle, on the CPU.
"""
import os

import numpy as np
import pytest

import oracle
import test_oracle_dispatch_combine as tdc
import test_oracle_expert_combine as tec
import test_oracle_expert_combine_fp8 as tef
import test_oracle_fp8 as tf8
import test_oracle_layout as tlay
import test_oracle_ll as tll

MUTANTS = {
    "padding rounds up a full segment": (
        "int32_t padded = ((c + A - 1) / A) * A;", "int32_t padded = (c / A + 1) * A;"),
    "offsets not accumulated": (
        "expert_offsets[e + 1] = expert_offsets[e] + padded;", "expert_offsets[e + 1] = padded;"),
    "rank of an expert by modulo": ("if (e >= 0 && e / L == r) in = 1;", "if (e >= 0 && e % R == r) in = 1;"),
    "masked slot counted": ("            if (e >= 0) num_tokens_per_expert[e] += 1;",
                            "            num_tokens_per_expert[e < 0 ? 0 : e] += 1;"),
    "tokens appended in reverse order": (
        "cursor[e] = expert_offsets[e];\n    for (int32_t t = 0; t < T; ++t) {",
        "cursor[e] = expert_offsets[e];\n    for (int32_t t = T - 1; t >= 0; --t) {"),
    "slot recorded as token": ("row_slot[r] = k;", "row_slot[r] = t;"),
    "ties rounded away from zero": ("if (d > 0.5f) return n + 1;", "if (d >= 0.5f) return n + 1;"),
    "no saturation (NaN code)": (
        "if (a >= 448.0f) return (uint8_t)(sign | 0x7E);", "if (a >= 448.0f) return (uint8_t)(sign | 0x7F);"),
    "subnormal step 2^-8": ("round_half_even_u(a * 512.0f)", "round_half_even_u(a * 256.0f)"),
    "exponent bias off by one": ("((uint32_t)(e + 7) << 3) | m", "((uint32_t)(e + 8) << 3) | m"),
    "amax without abs": (
        "amax = fmaxf(amax, fabsf(bf16_bits_to_float(xb[j])));",
        "amax = fmaxf(amax, bf16_bits_to_float(xb[j]));"),
    "scale stored inverted": ("scale[b] = amax_floor / 448.0f;", "scale[b] = 448.0f / amax_floor;"),
    "quantised with the dequant scale": (
        "float v = bf16_bits_to_float(xb[j]) * inv;", "float v = bf16_bits_to_float(xb[j]) * (amax_floor / 448.0f);"),
    "combine uses weight of k=0": (
        "double wk = (double)w[(int64_t)t * K + k];", "double wk = (double)w[(int64_t)t * K];"),
    "combine reads row of k=0": (
        "int32_t r = pos[(int64_t)t * K + k];\n            if (r == -1) continue;",
        "int32_t r = pos[(int64_t)t * K];\n            if (r == -1) continue;"),
    "combine drops the last k": ("for (int32_t k = 0; k < K; ++k) {\n            int32_t r = pos",
                                 "for (int32_t k = 0; k < K - 1; ++k) {\n            int32_t r = pos"),
    "dispatch copies the previous token": (
        "memcpy(dst, x + (int64_t)t * H, sizeof(uint16_t) * (size_t)H);",
        "memcpy(dst, x + (int64_t)(t > 0 ? t - 1 : 0) * H, sizeof(uint16_t) * (size_t)H);"),
    "low-latency slot not advanced": ("            recv_count[e] += 1;\n", "\n"),
    "low-latency overflow off by one": ("if (recv_count[e] >= M)", "if (recv_count[e] > M)"),
    "low-latency expert stride": ("pos[i] = (int32_t)((int64_t)e * M + recv_count[e]);",
                                  "pos[i] = (int32_t)((int64_t)e * (M - 1) + recv_count[e]);"),
    "low-latency masked slot counted": (
        "if (e < 0) { pos[i] = -1; continue; }              /* masked slot */",
        "if (e < 0) { pos[i] = -1; recv_count[0] += 1; continue; }"),
    "expert matrix transposed": ("* (double)bf16_bits_to_float(we[(int64_t)n * I + i]);",
                                 "* (double)bf16_bits_to_float(we[(int64_t)i * N + n]);"),
    "expert taken from k = 0": (
        "int64_t e = topk_idx[(int64_t)t * K + k];\n            int32_t r = pos[(int64_t)t * K + k];\n"
        "            if (e == -1 || r == -1) continue;\n"
        "            if (e < 0 || e >= E || r < 0 || r >= rows) return ORACLE_BAD_ARG;\n"
        "            const uint16_t *a",
        "int64_t e = topk_idx[(int64_t)t * K];\n            int32_t r = pos[(int64_t)t * K + k];\n"
        "            if (e == -1 || r == -1) continue;\n"
        "            if (e < 0 || e >= E || r < 0 || r >= rows) return ORACLE_BAD_ARG;\n"
        "            const uint16_t *a"),
    "gemm weight of the wrong slot": (
        "double wk = (double)topk_w[(int64_t)t * K + k];\n            for (int32_t n = 0; n < N; ++n) {\n"
        "                double acc = 0.0;\n                for (int32_t i = 0; i < I; ++i)\n",
        "double wk = (double)topk_w[(int64_t)t * K + (K - 1 - k)];\n            for (int32_t n = 0; n < N; ++n) {\n"
        "                double acc = 0.0;\n                for (int32_t i = 0; i < I; ++i)\n"),
    "fp8 gemm: expert taken from k = 0": (
        "            const uint8_t *we = w_q + (int64_t)e * N * I;",
        "            const uint8_t *we = w_q + (int64_t)topk_idx[(int64_t)t * K] * N * I;"),
    "fp8 gemm: weight of the wrong slot": (
        "double wk = (double)topk_w[(int64_t)t * K + k];\n            for (int32_t n = 0; n < N; ++n) {\n"
        "                double acc = 0.0;\n                for (int32_t i = 0; i < I; ++i) {\n",
        "double wk = (double)topk_w[(int64_t)t * K + (K - 1 - k)];\n            for (int32_t n = 0; n < N; ++n) {\n"
        "                double acc = 0.0;\n                for (int32_t i = 0; i < I; ++i) {\n"),
    "e4m3 value: exponent bias off by one": ("ldexp(8.0 + (double)m, e - 10)", "ldexp(8.0 + (double)m, e - 9)"),
    "e4m3 value: subnormal step 2^-8": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -8);"),
    "fp8 gemm: row scale of block 0": ("(double)act_scale[(int64_t)r * IB + b];", "(double)act_scale[(int64_t)r * IB];"),
    "fp8 gemm: column-major scale read row-major": (
        "(double)act_scale[(int64_t)b * scale_ld + r]", "(double)act_scale[(int64_t)r * IB + b]"),
    "fp8 gemm: expert block scale transposed": (
        "se[(int64_t)(n / 128) * IB + b]", "se[(int64_t)b * NB + n / 128]"),
    "fp8 gemm: expert block scale dropped": (
        "(value[we[(int64_t)n * I + i]] * sw)", "(value[we[(int64_t)n * I + i]] + 0.0 * sw)"),
    "padding row not zeroed": (
        "            memset(dst, 0, sizeof(uint16_t) * (size_t)H);\n",
        "            memset(dst, 0, sizeof(uint16_t) * (size_t)(H / 2));\n"),
}


def small_bruteforce(lib):
    for T in range(0, 3):
        for E in (1, 2, 4):
            for K in (1, 2):
                for flat in np.ndindex(*([E] * (T * K))) if T * K else [()]:
                    idx = np.array(flat, dtype=np.int64).reshape(T, K)
                    for R in [d for d in range(1, E + 1) if E % d == 0]:
                        for A in (1, 3):
                            L = lib.layout(idx, E, R, A)
                            ref = tlay.naive_layout(idx, E, R, A)
                            assert L.status == 0
                            for key, val in ref.items():
                                np.testing.assert_array_equal(
                                    getattr(L, key), np.asarray(val).reshape(getattr(L, key).shape))


PINS = [
    ("worked example", lambda lib: tlay.test_worked_example(lib)),
    ("brute force", small_bruteforce),
    ("invariants tiny", lambda lib: tlay.test_invariants_on_workloads(lib, "tiny")),
    ("invariants skew", lambda lib: tlay.test_invariants_on_workloads(lib, "skew")),
    ("e4m3 known codes", lambda lib: tf8.test_known_codes(lib)),
    ("e4m3 round trip", lambda lib: tf8.test_representable_values_round_trip(lib)),
    ("e4m3 brute force", lambda lib: tf8.test_brute_force_all_bf16(lib)),
    ("e4m3 ties", lambda lib: tf8.test_ties_and_neighbours(lib)),
    ("identity round trip", lambda lib: tdc.test_identity_round_trip(lib, 4)),
    ("masked slots", lambda lib: tlay.test_masked_slots(lib)),
    ("masked round trip", lambda lib: tdc.test_masked_slots_round_trip(lib)),
    ("one-hot", lambda lib: tdc.test_one_hot_selects_expert_row(lib)),
    ("lesson exercise", lambda lib: tdc.test_lesson_exercise_restated(lib)),
    ("fp8 properties", lambda lib: tdc.test_fp8_dispatch_properties(lib, 5)),
    ("gemm scaled identity", lambda lib: tec.test_scaled_identity_experts(lib)),
    ("gemm rank one", lambda lib: tec.test_rank_one_experts(lib)),
    ("gemm masked", lambda lib: tec.test_masked_slots_and_selection(lib)),
    ("fp8 gemm decoder", lambda lib: tef.test_e4m3_decoder_all_codes(lib)),
    ("fp8 gemm unit scales", lambda lib: tef.test_unit_scales_reduce_to_bf16_gemm(lib)),
    ("fp8 gemm block scales", lambda lib: tef.test_block_scales_closed_form(lib)),
    ("fp8 gemm column-major", lambda lib: tef.test_column_major_scales(lib)),
    ("fp8 gemm masked", lambda lib: tef.test_masked_slots_and_selection_fp8(lib)),
    ("ll worked example", lambda lib: tll.test_ll_worked_example(lib)),
    ("ll brute force", lambda lib: tll.test_ll_bruteforce_tiny(lib)),
    ("ll round trip", lambda lib: tll.test_ll_round_trip(lib)),
]


def run_pins(lib):
    failed = []
    for name, fn in PINS:
        try:
            fn(lib)
        except Exception:  # noqa: BLE001 - any failure of a pin counts
            failed.append(name)
    return failed


def test_unmutated_source_passes_battery(tmp_path):
    so = oracle.compile_source(oracle.source_text(), str(tmp_path / "orig.so"))
    with oracle.use_library(so):
        assert run_pins(oracle) == []


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor not unique: {name}"
    so = oracle.compile_source(src.replace(old, new), str(tmp_path / "mutant.so"))
    with oracle.use_library(so):
        failed = run_pins(oracle)
    assert failed, f"no pin caught the mutant '{name}'"
