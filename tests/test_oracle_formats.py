"""Pins of the oracle's number formats against things other than itself.

- E2M1 decode: the sixteen values of the FP4 E2M1 format, written out.
- E4M3 decode: torch's float8_e4m3fn conversion (a library routine).
- Both encoders: a brute-force nearest-value search with ties to the even
  code (written here, independently of the oracle's table scan), a threshold
  rule for E2M1, and torch's RNE float8_e4m3fn cast on [0, 448].
- Scale formulas: exact rational arithmetic (correct rounding of a quotient).

NVFP4 is E2M1 data with E4M3 block scales and an FP32 second-level scale
(TransformerEngine #2931 "Implement per-token NVFP4 fprop recipe", Changes;
sequence diagram: FP4 data, FP8 scales, amax vector).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
               -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
FLT_MAX = np.finfo(np.float32).max


def f32_bits(v):
    return np.asarray(v, dtype=np.float32).view(np.uint32)


def from_bits(b):
    return np.asarray(b, dtype=np.uint32).view(np.float32)


# ------------------------------------------------------------------ decode

def test_e2m1_decode_all_16_codes():
    for code, want in enumerate(E2M1_VALUES):
        got = oracle.e2m1_decode(code)
        assert got == want and np.signbit(got) == np.signbit(want), (code, got, want)


def test_e4m3_decode_all_256_codes_vs_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    for c in range(256):
        got = np.float32(oracle.e4m3_decode(c))
        if np.isnan(ref[c]):
            assert np.isnan(got), c
            assert c in (0x7F, 0xFF)
        else:
            assert got == ref[c] and np.signbit(got) == np.signbit(ref[c]), (c, got, ref[c])
    # the format's landmarks
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6


# ------------------------------------------------------- brute-force search

def brute_nearest(a: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest table entry to each a >= 0; ties to the even
    index. Distances in float64 (exact for the neighbours that matter)."""
    out = np.empty(a.shape, dtype=np.int64)
    t = table.astype(np.float64)
    for s in range(0, a.size, 20000):
        blk = a[s:s + 20000].astype(np.float64)
        d = np.abs(blk[:, None] - t[None, :])
        dmin = d.min(axis=1, keepdims=True)
        cand = d == dmin
        idx = np.arange(t.size)[None, :]
        # if two candidates tie, prefer the even index
        even = cand & (idx % 2 == 0)
        has_even = even.any(axis=1)
        first = np.argmax(cand, axis=1)
        first_even = np.argmax(even, axis=1)
        out[s:s + 20000] = np.where(has_even, first_even, first)
    return out


def sweep(lo: float, hi: float, landmarks, window=2048, stride=4099):
    """All fp32 bit patterns within +-window ulps of each landmark, plus a
    strided sweep over [lo, hi]."""
    parts = [np.arange(f32_bits(lo), f32_bits(hi) + 1, stride, dtype=np.int64)]
    for m in landmarks:
        b = int(f32_bits(m))
        parts.append(np.arange(max(b - window, 0), b + window + 1, dtype=np.int64))
    bits = np.unique(np.concatenate(parts))
    bits = bits[(bits >= 0) & (bits < 0x7F800000)]
    return from_bits(bits.astype(np.uint32))


E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def e2m1_by_thresholds(y: np.ndarray) -> np.ndarray:
    """Second, independent E2M1 encoder: threshold comparisons with the ties
    (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) sent to the even code."""
    a = np.abs(y)
    mag = np.select(
        [a <= 0.25, a < 0.75, a <= 1.25, a < 1.75, a <= 2.5, a < 3.5, a <= 5.0],
        [0, 1, 2, 3, 4, 5, 6], default=7)
    return (mag | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def test_e2m1_encode_vs_brute_force_and_thresholds():
    mids = (E2M1_MAG[1:] + E2M1_MAG[:-1]) / 2
    y = sweep(0.0, 8.0, list(mids) + list(E2M1_MAG[1:]) + [1e-30])
    got = oracle.e2m1_encode(y)
    want = brute_nearest(y, E2M1_MAG).astype(np.uint8)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got, e2m1_by_thresholds(y))
    # negatives: same magnitude code with the sign bit
    gn = oracle.e2m1_encode(-y)
    np.testing.assert_array_equal(gn, want | 8)


@pytest.mark.parametrize("y,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    (6.0, 7), (7.0, 7), (1e30, 7), (float("inf"), 7), (0.0, 0), (-0.0, 8),
    (-1e-20, 8), (-0.25, 8), (-0.2500001, 9), (-6.5, 15)])
def test_e2m1_encode_ties_sign_saturation(y, code):
    assert int(oracle.e2m1_encode(np.array([y], np.float32))[0]) == code


def e4m3_table():
    return np.array([oracle.e4m3_decode(c) for c in range(127)], dtype=np.float32)


def test_e4m3_encode_vs_brute_force():
    t = e4m3_table()
    mids = (t[1:] + t[:-1]) / 2
    v = sweep(0.0, 480.0, list(mids) + list(t[1:]) + [1e-30, 2.0 ** -10])
    got = oracle.e4m3_encode(v)
    want = brute_nearest(v, t).astype(np.uint8)
    np.testing.assert_array_equal(got, want)


def test_e4m3_encode_vs_torch_rne_on_0_448():
    t = e4m3_table()
    mids = (t[1:] + t[:-1]) / 2
    v = sweep(0.0, 448.0, list(mids), window=512, stride=8191)
    v = v[v <= 448.0]
    ref = torch.from_numpy(v.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(v), ref)


@pytest.mark.parametrize("v,code", [
    (448.0, 0x7E), (448.5, 0x7E), (464.0, 0x7E), (480.0, 0x7E), (1e30, 0x7E),
    (float(FLT_MAX), 0x7E), (float("inf"), 0x7E),
    (2.0 ** -10, 0x00), (np.nextafter(np.float32(2.0 ** -10), np.float32(1)), 0x01),
    (3 * 2.0 ** -10, 0x02), (0.0, 0x00), (-0.0, 0x80), (88.0, 0x6B), (92.0, 0x6C), (91.99999, 0x6B),
    (92.00001, 0x6C)])
def test_e4m3_encode_saturation_and_ties(v, code):
    assert int(oracle.e4m3_encode(np.array([v], np.float32))[0]) == code


# ------------------------------------------------------------ scale rounding

def rn_f32(q: Fraction) -> np.float32:
    """The float32 nearest to the rational q (ties to even mantissa), found
    by comparing exact distances of the candidates around float(q)."""
    f = np.float32(float(q))
    cands = {f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))}
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - q)
        key = (d, int(f32_bits(c)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def test_second_level_scales_are_correctly_rounded_quotients():
    rng = np.random.default_rng(7)
    a = np.concatenate([
        (rng.integers(1, 0x7F7F, 3000, dtype=np.uint32) << 16).view(np.float32),  # bf16 values
        np.float32([6.0, 5.0, 2688.0, 1.0, 448.0, 3.0e38, 1e-30])])
    for ai in a:
        ai = np.float32(ai)
        q = Fraction(2688) / Fraction(float(ai))
        want = rn_f32(q) if q <= Fraction(float(FLT_MAX)) else None
        got = oracle.s_enc(ai)
        if want is None or not np.isfinite(want):
            # quotient above the float range: clamped
            assert got == FLT_MAX
        else:
            assert got == want, (ai, got, want)
        assert oracle.s_dec(ai) == rn_f32(Fraction(float(ai)) / 2688)


def test_second_level_special_cases():
    assert oracle.s_enc(0.0) == 1.0
    assert oracle.s_dec(0.0) == 0.0
    assert oracle.s_enc(6.0) == 448.0
    assert oracle.s_enc(2688.0) == 1.0
    assert oracle.s_dec(2688.0) == 1.0
    tiny = from_bits(np.uint32(1 << 16))  # smallest positive bf16 (subnormal)
    assert oracle.s_enc(float(tiny)) == FLT_MAX
