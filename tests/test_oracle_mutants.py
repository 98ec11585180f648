"""The oracle's pins must catch plausible mistakes.

Each mutant below is the oracle's C source with one plausible slip planted in
it (a wrong constant, a tie sent the wrong way, swapped nibbles, a transposed
index, a lost sign). Every mutant is compiled on the CPU into a temporary
library, swapped in for the real oracle, and the pin battery of
test_oracle_formats.py / test_oracle_blocks.py must fail on it. The real
oracle is restored afterwards. Nothing here touches a GPU.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild

from . import test_oracle_blocks as tb
from . import test_oracle_formats as tf

SRC = open(obuild.SRC).read()

MUTANTS = {
    "block_div_4": ("float t = bmax / 6.0f;", "float t = bmax / 4.0f;"),
    "senc_constant": ("float q = 2688.0f / a;", "float q = 2687.0f / a;"),
    "ties_to_odd": ("return (c % 2 == 0) ? c : c + 1;", "return (c % 2 == 1) ? c : c + 1;"),
    "ties_down": ("if (below < above) return c;", "if (below <= above) return c;"),
    "row_nibbles_swapped": (
        "row_data[r * (K / 2) + 8 * b + j] =\n              (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));",
        "row_data[r * (K / 2) + 8 * b + j] =\n              (uint8_t)(codes[2 * j + 1] | (codes[2 * j] << 4));"),
    "col_scale_transposed": ("gscale[k * (m / 16) + b] = s8;", "gscale[b * K + k] = s8;"),
    "col_rows_reversed": ("blk[j] = nvo_bf16_to_f32(x[(o + 16 * b + j) * K + k]);",
                          "blk[j] = nvo_bf16_to_f32(x[(o + 16 * b + (15 - j)) * K + k]);"),
    "negative_zero_unsigned": ("uint8_t sign = signbit(y) ? 0x8 : 0x0;",
                               "uint8_t sign = (y < 0.0f) ? 0x8 : 0x0;"),
    "sdec_constant": ("float nvo_s_dec(float a) { return a / 2688.0f; }",
                      "float nvo_s_dec(float a) { return a / 448.0f; }"),
    "col_amax_index": ("col_amax[(int64_t)g * K + k] = m;", "col_amax[k * E + g] = m;"),
    "element_scale_skew": ("float y = x16[j] * enc;", "float y = x16[j] * enc * 1.0001f;"),
    "e4m3_bias": ("mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);",
                  "mag = ldexpf(1.0f + (float)m / 8.0f, e - 8);"),
    "e2m1_exponent": ("ldexpf(1.0f + 0.5f * (float)m, e - 1)", "ldexpf(1.0f + 0.5f * (float)m, e - 2)"),
    "dequant_nibbles": ("(c % 2 == 0) ? (byte & 0xF) : (byte >> 4)",
                        "(c % 2 == 0) ? (byte >> 4) : (byte & 0xF)"),
    "zero_scale_not_guarded": ("if (sc != 0) {", "if (1) {"),
    "zero_amax_scale": ("if (a == 0.0f) return 1.0f;", "if (a == 0.0f) return 0.0f;"),
    "block_max_skips_last": ("for (int j = 0; j < 16; j++) {\n    float ax = fabsf(x16[j]);",
                             "for (int j = 0; j < 15; j++) {\n    float ax = fabsf(x16[j]);"),
    "row_amax_skips_sign": ("float a = fabsf(nvo_bf16_to_f32(x[r * K + k]));\n        if (a > m) m = a;\n      }\n      row_amax[r] = m;",
                            "float a = nvo_bf16_to_f32(x[r * K + k]);\n        if (a > m) m = a;\n      }\n      row_amax[r] = m;"),
}


def battery():
    """The pins, cheapest first; each entry raises on a detected mistake."""
    yield lambda: tf.test_e2m1_decode_all_16_codes()
    yield lambda: tf.test_e4m3_decode_all_256_codes_vs_torch()
    yield lambda: tf.test_second_level_special_cases()
    for v, c in [(0.25, 0), (0.75, 2), (2.5, 4), (5.0, 6), (-0.0, 8), (-1e-20, 8), (7.0, 7)]:
        yield lambda v=v, c=c: tf.test_e2m1_encode_ties_sign_saturation(v, c)
    for v, c in [(92.0, 0x6C), (3 * 2.0 ** -10, 0x02), (464.0, 0x7E), (88.0, 0x6B)]:
        yield lambda v=v, c=c: tf.test_e4m3_encode_saturation_and_ties(v, c)
    yield lambda: tb.test_hand_worked_blocks_rowwise("block_a")
    yield lambda: tb.test_hand_worked_blocks_rowwise("block_b")
    yield lambda: tb.test_hand_worked_block_a_colwise_and_dequant()
    yield lambda: tb.test_zero_rows_and_empty_groups()
    yield lambda: tb.test_block_whose_scale_rounds_to_zero_encodes_signed_zeros()
    for args in [(12, 32, [16, 0, 32], "wide"), (15, 128, [32, 64, 0, 32], "wide"),
                 (13, 64, [48, 16], "heavy")]:
        yield lambda args=args: tb.test_second_encoder_agrees_on_tiny_inputs(*args)
    for d in ["normal", "wide", "heavy"]:
        yield lambda d=d: tb.test_invariants_rowwise_and_colwise(d)
    yield lambda: tf.test_second_level_scales_are_correctly_rounded_quotients()
    yield lambda: tf.test_e4m3_encode_vs_brute_force()
    yield lambda: tf.test_e2m1_encode_vs_brute_force_and_thresholds()


def test_every_mutation_site_exists():
    for name, (old, new) in MUTANTS.items():
        assert SRC.count(old) == 1, name


@pytest.fixture(scope="module")
def mutant_dir():
    with tempfile.TemporaryDirectory() as d:
        # the unmutated oracle's header must sit next to each mutant source
        with open(os.path.join(d, "nvfp4_oracle.h"), "w") as f:
            f.write(open(os.path.join(obuild.HERE, "nvfp4_oracle.h")).read())
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_dir):
    old, new = MUTANTS[name]
    src = os.path.join(mutant_dir, name + ".c")
    so = os.path.join(mutant_dir, name + ".so")
    with open(src, "w") as f:
        f.write(SRC.replace(old, new))
    subprocess.run(["gcc", *obuild.CFLAGS, "-o", so, src, "-lm"], check=True,
                   capture_output=True)
    saved = oracle.lib()
    oracle._lib = oracle.load(so)
    try:
        caught = None
        for check in battery():
            try:
                check()
            except (AssertionError, oracle.OracleError, ValueError) as e:
                caught = e
                break
        assert caught is not None, f"no pin detects mutant {name}"
    finally:
        oracle._lib = saved
