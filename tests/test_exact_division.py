"""The CUDA kernels replace two IEEE divisions per block by Markstein's
correction (P. Markstein, "Computation of elementary functions on the IBM
RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with y = RN(1/b),

    q0 = RN(a * y);  r = fma(-q0, b, a);  q = fma(r, y, q0)

and the kernels rely on q == RN(a / b) (RN = binary32, nearest even). This
test proves that exhaustively for every operand the kernels can meet, with
each binary32 operation emulated exactly in integer arithmetic:

- block max / 6: a = every positive finite bf16 value >= 2^-100 (smaller
  maxima take the kernels' exact-division fallback), b = 6;
- element scale S_enc / e4m3(s8): a = S_enc(amax) for every positive finite
  bf16 amax with S_enc >= 2^-100 (the rest take the fallback), b = every
  E4M3 significand. Scaling b by a power of two scales y, q0, r and q by the
  inverse power exactly (every intermediate stays normal: r is about
  a * 2^-24 >= 2^-124), so the eight E4M3 significands 1, 1.125, .., 1.875
  cover all 126 positive E4M3 values.
Overflow of q0 only happens when the true quotient is at least FLT_MAX, and
the kernels then clamp to FLT_MAX like the oracle; it is excluded here.
"""
import struct

import numpy as np

FLT_MAX = float(np.finfo(np.float32).max)


def split(x: float):
    """positive normal binary32 -> (m, e): x = m * 2^e, 2^23 <= m < 2^24"""
    b = struct.unpack("<I", struct.pack("<f", x))[0]
    ex = (b >> 23) & 0xFF
    assert 0 < ex < 255, x
    return (b & 0x7FFFFF) | 0x800000, ex - 150


def rn(n: int, e: int):
    """Round the positive value n * 2^e to 24 significant bits, ties to even.
    n may carry a sticky bit below the rounding position."""
    sh = n.bit_length() - 24
    if sh <= 0:
        return n << -sh, e + sh
    q, rem = n >> sh, n & ((1 << sh) - 1)
    half = 1 << (sh - 1)
    if rem > half or (rem == half and (q & 1)):
        q += 1
    if q >> 24:
        q >>= 1
        sh += 1
    return q, e + sh


def rn_div(am, ae, bm, be):
    """RN((am 2^ae) / (bm 2^be))"""
    k = 50
    q, r = divmod(am << k, bm)
    return rn((q << 1) | (1 if r else 0), ae - be - k - 1)


def markstein(am, ae, bm, be, ym, ye):
    q0m, q0e = rn(am * ym, ae + ye)
    # r = a - q0*b, exact in integers; the fma returns RN of it, which must be exact
    e0 = min(ae, q0e + be)
    R = (am << (ae - e0)) - ((q0m * bm) << (q0e + be - e0))
    if R != 0:
        rm, re = rn(abs(R), e0)
        assert (rm << (re - e0) if re >= e0 else rm >> (e0 - re)) == abs(R), "fma remainder inexact"
    # q = RN(q0 + r*y), from the exact sum
    e1 = min(q0e, e0 + ye)
    T = (q0m << (q0e - e1)) + ((R * ym) << (e0 + ye - e1))
    assert T > 0
    return rn(T, e1)


def f32(x):
    return float(np.float32(x))


def bf16_values():
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    return [float(v) for v in (bits << 16).view(np.float32)]


def test_integer_emulation_matches_binary32():
    rng = np.random.default_rng(3)
    a = rng.integers(0x00800000, 0x7E000000, 5000, dtype=np.uint32).view(np.float32)
    b = rng.integers(0x20000000, 0x5F000000, 5000, dtype=np.uint32).view(np.float32)
    with np.errstate(over="ignore", under="ignore"):
        q = (a / b).astype(np.float32)
        p = (a * (b / np.float32(1e8))).astype(np.float32)
    for ai, bi, qi, pi in zip(a, b, q, p):
        if 1e-37 < qi < 1e37:
            m, e = rn_div(*split(float(ai)), *split(float(bi)))
            assert m * 2.0 ** e == float(qi)
        bi8 = float(np.float32(bi / np.float32(1e8)))
        if 1e-37 < pi < 1e37:
            m, e = rn(split(float(ai))[0] * split(bi8)[0], split(float(ai))[1] + split(bi8)[1])
            assert m * 2.0 ** e == float(pi)


def test_block_max_over_6():
    bm, be = split(6.0)
    ym, ye = split(f32(np.float32(1) / np.float32(6)))
    n = 0
    for a in bf16_values():
        if a < 2.0 ** -100:
            continue
        am, ae = split(a)
        assert markstein(am, ae, bm, be, ym, ye) == rn_div(am, ae, bm, be), a
        n += 1
    assert n == 29184  # 228 binades (2^-100 .. 2^127) x 128 significands


def test_element_scale_over_e4m3():
    senc = set()
    for a in bf16_values():
        s = f32(min(f32(np.float32(2688.0) / np.float32(a)), FLT_MAX)) if a > 0 else 1.0
        if s >= 2.0 ** -100:
            senc.add(s)
    senc.add(1.0)
    sig = [1 + k / 8 for k in range(8)]  # E4M3 significands
    n = 0
    for v in sig:
        bm, be = split(v)
        ym, ye = split(f32(np.float32(1) / np.float32(v)))
        for s in senc:
            if s / v >= FLT_MAX * (1 - 2.0 ** -22) or s * (1 / v) >= FLT_MAX * (1 - 2.0 ** -22):
                continue  # overflow: the kernels clamp to FLT_MAX
            am, ae = split(s)
            assert markstein(am, ae, bm, be, ym, ye) == rn_div(am, ae, bm, be), (s, v)
            n += 1
    assert n > 200000


def test_tiny_block_under_fast_range_amax_has_zero_scale():
    """The kernels use the shortcuts for every block of a tile whose row and
    column amax values are 0 or in [2^-81, 2^111]. A block maximum below
    2^-100 is outside the divide-by-6 proof, but under such an amax its
    block scale is E4M3 zero however b/6 rounds: the largest such scale,
    from the largest bf16 below 2^-100 under amax 2^-81, is below 2^-10,
    the smallest value that does not round to E4M3 zero."""
    b = np.float32(np.uint32(0x0D7F0000).view(np.float32))  # largest bf16 < 2^-100
    a = np.float32(2.0 ** -81)
    senc = np.float32(2688.0) / a
    for t in (np.float32(b / np.float32(6)), np.nextafter(np.float32(b / np.float32(6)), np.float32(1))):
        s32 = np.float32(t * senc)
        assert s32 < np.float32(2.0 ** -10) * np.float32(0.9)
    # and the upper end: S_enc of the largest fast-path amax is still >= 2^-100
    assert np.float32(2688.0) / np.float32(2.0 ** 111) >= np.float32(2.0 ** -100)
