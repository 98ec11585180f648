"""Pins of the oracle's consumer-side functions (no GPU).

- the 128x4-tiled scale layout: byte positions worked out by hand from the
  index map, tile order, zero padding, and that it is a permutation;
- bfloat16 round-to-nearest-even: hand-made bit patterns (exact, below and
  above half an ulp, ties to even both ways, overflow to infinity, signed
  zero, subnormals, NaN), and agreement with torch's own conversion on random
  values (a library routine of the same definition);
- the post-GEMM row scaling (TransformerEngine #2931, sequence diagram):
  exact products, the bias added after the scaling, one rounding each.
"""
import struct

import numpy as np
import pytest
import torch

import oracle


def f32(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", bits))[0]


@pytest.mark.parametrize("r,c,pos", [
    (0, 0, 0), (0, 3, 3), (1, 0, 16), (31, 0, 496), (32, 0, 4), (33, 2, 22),
    (64, 1, 9), (96, 3, 15), (127, 3, 511), (100, 2, 4 * 16 + 3 * 4 + 2),
])
def test_swizzle_positions_inside_one_tile(r, c, pos):
    s = np.zeros((128, 4), dtype=np.uint8)
    s[r, c] = 0xAB
    out = oracle.swizzle_scales_128x4(s, 128, 4)
    assert out.size == 512
    assert list(np.nonzero(out)[0]) == [pos]


def test_swizzle_tile_order_is_row_major_over_tiles():
    # [256, 8]: four tiles; tile (ti, tj) starts at byte 512 * (2 * ti + tj)
    s = np.zeros((256, 8), dtype=np.uint8)
    s[0, 4] = 1    # tile (0, 1), local (0, 0)
    s[128, 0] = 2  # tile (1, 0), local (0, 0)
    s[129, 5] = 3  # tile (1, 1), local (1, 1) -> 16 + 1
    out = oracle.swizzle_scales_128x4(s, 256, 8)
    assert out[512] == 1 and out[1024] == 2 and out[1536 + 17] == 3
    assert np.count_nonzero(out) == 3


def test_swizzle_pads_partial_tiles_with_zeros():
    rows, cols = 130, 5
    s = np.full((rows, cols), 7, dtype=np.uint8)
    out = oracle.swizzle_scales_128x4(s, rows, cols)
    assert out.size == 256 * 8
    assert np.count_nonzero(out) == rows * cols
    # tile (1, 1) holds only element (128, 4) and (129, 4)
    t11 = out[3 * 512:4 * 512]
    assert np.count_nonzero(t11) == 2 and t11[0] == 7 and t11[16] == 7


def test_swizzle_is_a_permutation_on_whole_tiles():
    g = np.random.default_rng(3)
    rows, cols = 384, 12
    vals = g.permutation(rows * cols).astype(np.int64)
    # unique values need more than 8 bits: swizzle the low and high bytes separately
    lo = (vals & 0xFF).astype(np.uint8).reshape(rows, cols)
    hi = (vals >> 8).astype(np.uint8).reshape(rows, cols)
    slo = oracle.swizzle_scales_128x4(lo, rows, cols).astype(np.int64)
    shi = oracle.swizzle_scales_128x4(hi, rows, cols).astype(np.int64)
    assert sorted((shi << 8) | slo) == sorted(vals)


@pytest.mark.parametrize("bits,want", [
    (0x3F800000, 0x3F80),   # 1.0, exact
    (0x3F808000, 0x3F80),   # tie, kept part even: down
    (0x3F818000, 0x3F82),   # tie, kept part odd: up
    (0x3F807FFF, 0x3F80),   # just below half: down
    (0x3F808001, 0x3F81),   # just above half: up
    (0xBF80C000, 0xBF81),   # negative, above half: magnitude up
    (0x7F7FFFFF, 0x7F80),   # largest float rounds to infinity
    (0x7F800000, 0x7F80),   # infinity
    (0x80000000, 0x8000),   # negative zero
    (0x00008000, 0x0000),   # subnormal tie to even (0)
    (0x00018000, 0x0002),   # subnormal tie to even (up)
])
def test_bf16_round_to_nearest_even(bits, want):
    assert oracle.f32_to_bf16(f32(bits)) == want


def test_bf16_nan_stays_nan():
    b = oracle.f32_to_bf16(f32(0x7FC00001))
    assert (b & 0x7F80) == 0x7F80 and (b & 0x7F) != 0
    b = oracle.f32_to_bf16(f32(0x7F800001))  # a NaN whose payload is all in the dropped bits
    assert (b & 0x7F80) == 0x7F80 and (b & 0x7F) != 0


def test_bf16_matches_torch_conversion_on_random_values():
    g = np.random.default_rng(5)
    v = (g.standard_normal(20000) * np.exp2(g.integers(-130, 128, 20000))).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_post_scale_exact_cases():
    x = np.array([[1.5, -2.0, 0.0, 3.0], [1.0, 1.0, -1.0, 0.5]], dtype=np.float32)
    amax = np.array([2.0, 0.25], dtype=np.float32)
    f, b = oracle.row_post_scale(x, amax)
    assert np.array_equal(f, np.array([[3.0, -4.0, 0.0, 6.0], [0.25, 0.25, -0.25, 0.125]], np.float32))
    assert b[0, 0] == 0x4040 and b[0, 1] == 0xC080 and b[1, 3] == 0x3E00
    bias = np.array([1.0, 2.0, 3.0, 4.0], dtype=np.float32)
    f2, _ = oracle.row_post_scale(x, amax, bias)
    assert np.array_equal(f2, f + bias[None, :])


def test_post_scale_rounds_after_each_operation():
    # 1 + 2^-23 times 1 + 2^-23 is not a float: the product rounds first,
    # then adding the bias rounds again
    x = np.array([[f32(0x3F800001)]], dtype=np.float32)
    a = np.array([f32(0x3F800001)], dtype=np.float32)
    f, _ = oracle.row_post_scale(x, a)
    assert struct.unpack("<I", struct.pack("<f", float(f[0, 0])))[0] == 0x3F800002
    f2, _ = oracle.row_post_scale(x, a, np.array([-1.0], np.float32))
    assert float(f2[0, 0]) == 2.0 ** -22
