"""Pins of the oracle's MXFP4 functions (no GPU).

MXFP4 = E2M1 data, blocks of 32, one E8M0 power-of-two scale per block
(TransformerEngine #3824, Testing: "E2M1/block-32/E8M0"); the scale rule is
the OCP Microscaling conversion (shared exponent floor(log2 amax) - 2,
clamped to the E8M0 range). Pinned by hand-worked blocks, exact round trips
of representable blocks, the error bound of the encoding, and the identity
between the colwise output and the rowwise output of each group's transpose.
"""
import math

import numpy as np
import pytest

import oracle
from nvfp4_row_scaled_b200 import workloads

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


@pytest.mark.parametrize("code,value", [(127, 1.0), (128, 2.0), (126, 0.5), (0, 2.0 ** -127),
                                        (254, 2.0 ** 127), (137, 1024.0)])
def test_e8m0_decode(code, value):
    assert oracle.e8m0_decode(code) == value


def test_e8m0_ff_is_nan():
    assert math.isnan(oracle.e8m0_decode(255))


def block(*vals):
    x = np.zeros(32, dtype=np.float32)
    x[:len(vals)] = vals
    return x


@pytest.mark.parametrize("vals,scale,codes", [
    ((6.0, -1.0, 0.75, 0.25), 127, [7, 0xA, 2, 0]),     # amax 6: scale 2^0; 0.75 ties to 1.0, 0.25 to 0
    ((7.0, 3.5), 127, [7, 6]),                           # 7 saturates to 6; 3.5 ties to 4
    ((8.0, -1.0, 0.75), 128, [6, 0x9, 1]),               # amax 8: scale 2^1
    ((1.5, 0.375), 125, [7, 3]),                         # amax 1.5: floor(log2) = 0, scale 2^-2
    ((5.9, 1.1), 127, [7, 2]),
    ((4.0, -4.0, 2.5), 127, [6, 0xE, 4]),                # 2.5 ties to 2 (even)
])
def test_block_hand_worked(vals, scale, codes):
    s8, c = oracle.mx_block_encode(block(*vals))
    assert s8 == scale
    assert list(c[:len(codes)]) == codes
    assert not c[len(codes):].any()


def test_zero_block_and_clamped_exponents():
    s8, c = oracle.mx_block_encode(np.zeros(32, np.float32))
    assert s8 == 0 and not c.any()
    s8, c = oracle.mx_block_encode(block(2.0 ** -130, -(2.0 ** -131)))
    assert s8 == 0                     # floor(log2) - 2 = -132 clamps to -127
    assert list(c[:2]) == [0, 0x8]     # 2^-3 and -2^-4 after scaling round to (signed) zero
    s8, c = oracle.mx_block_encode(block(1.5 * 2.0 ** 127))
    assert s8 == 127 + 125 and c[0] == 7  # 1.5 * 2^127 / 2^125 = 6, the code of 6


def test_representable_blocks_round_trip_exactly():
    g = np.random.default_rng(11)
    for _ in range(200):
        s = int(g.integers(-120, 120))
        codes = g.integers(0, 16, 32)
        codes[int(g.integers(0, 32))] = int(g.choice([6, 7, 14, 15]))  # |x| = 4 or 6 sets the exponent
        x = np.array([(-1.0 if c & 8 else 1.0) * E2M1[c & 7] * 2.0 ** s for c in codes], dtype=np.float32)
        s8, got = oracle.mx_block_encode(x)
        assert s8 == s + 127
        dq = oracle.mx_dequantize(np.array([got[i] | (got[i + 1] << 4) for i in range(0, 32, 2)], np.uint8),
                                  np.array([s8], np.uint8), 1, 32)[0]
        assert np.array_equal(dq, x)


def test_encoding_error_bound():
    """|x_hat - x| <= 2^s (half the widest E2M1 gap) below 6 * 2^s, and at
    most 2 * 2^s in the saturating range (6, 8) * 2^s."""
    g = np.random.default_rng(12)
    for _ in range(300):
        x = (g.standard_normal(32) * 2.0 ** float(g.integers(-20, 20))).astype(np.float32)
        s8, c = oracle.mx_block_encode(x)
        s = 2.0 ** (s8 - 127)
        xh = np.array([(-1.0 if k & 8 else 1.0) * E2M1[k & 7] for k in c]) * s
        err = np.abs(xh - x.astype(np.float64))
        sat = np.abs(x) > 6 * s
        assert np.all(err[~sat] <= s + 1e-30)
        assert np.all(err[sat] <= 2 * s)
        assert np.all((np.sign(xh) == np.sign(x)) | (xh == 0))


def test_colwise_is_the_rowwise_cast_of_each_group_transposed():
    w = workloads.random_case(13, 96, [64, 0, 32, 96], dist="wide")
    xb = workloads.bits(w.x)
    K = w.K
    out = oracle.mx_group_cast(xb, w.m_splits)
    o = 0
    for g, m in enumerate(w.m_splits):
        if m == 0:
            continue
        t = oracle.mx_group_cast(np.ascontiguousarray(xb[o:o + m].T), [K], rows=True, cols=False)
        assert np.array_equal(out["col_data"][K * o // 2:K * (o + m) // 2], t["row_data"].reshape(-1))
        assert np.array_equal(out["col_scale"][K * o // 32:K * (o + m) // 32], t["row_scale"].reshape(-1))
        o += m


def test_bad_arguments():
    x = np.zeros((64, 48), dtype=np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.mx_group_cast(x, [64])        # K % 32
    x = np.zeros((48, 64), dtype=np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.mx_group_cast(x, [16, 32])    # colwise needs groups of 32
    oracle.mx_group_cast(x, [16, 32], rows=True, cols=False)  # rowwise does not
