"""Pins of the oracle's block math, grouped layout and invariants.

- Hand-worked blocks (tests/golden/block_*.json, derived by hand).
- A second encoder written here with numpy (nearest-value search, torch's
  E4M3 table, numpy packing and transposes) on tiny inputs.
- Invariants that hold for any input: the dequantised magnitude never
  exceeds the governing amax, the per-element error is at most half an E2M1
  step times the block's scale, the block holding the amax gets scale 0x7E and
  code +-7, zero rows and empty groups give zeros.
- Brute-force amax; colwise output of a group equals the rowwise output of
  its transpose.

The grouped amax/cast structure is TransformerEngine #3649 ("single-launch
grouped row-scaled NVFP4 cast", Description); the per-token scales and the
dequantize row lookup are TransformerEngine #2931 ("Implement per-token NVFP4
fprop recipe", Changes, Important Files Changed, sequence diagram).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from nvfp4_row_scaled_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FLT_MAX = np.float32(np.finfo(np.float32).max)


def to_bits(v):
    a = np.asarray(v, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------- golden blocks

@pytest.mark.parametrize("name", ["block_a", "block_b"])
def test_hand_worked_blocks_rowwise(name):
    gb = json.load(open(os.path.join(GOLDEN, name + ".json")))
    K = gb["K"]
    row = np.array(gb["row"], dtype=np.float32)
    assert np.array_equal(to_bits(row).astype(np.uint32) << 16, row.view(np.uint32)), "bf16-exact"
    x = to_bits(row).reshape(1, K)
    ra, _ = oracle.group_amax(x, [1], cols=False)
    assert ra[0] == np.float32(gb["row_amax"])
    out = oracle.group_cast(x, [1], ra, None, cols=False)
    assert out["row_data"].tobytes().hex() == gb["data_hex"]
    assert [f"{b:02x}" for b in out["row_scale"].reshape(-1)] == gb["scale_bytes"]
    assert out["row_s2"][0] == np.float32(gb["row_amax"]) / np.float32(2688)


def test_hand_worked_block_a_colwise_and_dequant():
    gb = json.load(open(os.path.join(GOLDEN, "block_a.json")))
    col = np.array(gb["row"], dtype=np.float32)
    # the block as column 0 of a 16 x 16 group; other columns zero
    xf = np.zeros((16, 16), dtype=np.float32)
    xf[:, 0] = col
    x = to_bits(xf)
    ra, ca = oracle.group_amax(x, [16])
    assert ca[0] == 6.0 and np.all(ca[1:] == 0)
    out = oracle.group_cast(x, [16], ra, ca)
    cdata = oracle.col_slice(out["col_data"], [16], 16, 0, 2)
    cscale = oracle.col_slice(out["col_scale"], [16], 16, 0, 16)
    assert cdata[0].tobytes().hex() == gb["data_hex"]
    assert cscale[0, 0] == 0x7E
    assert np.all(cdata[1:] == 0) and np.all(cscale[1:] == 0)
    # dequantize: value(code) * 448 * fl(6/2688), one rounding
    xh = oracle.dequantize(cdata, cscale, out["col_s2"][:16], 16, 16)
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    codes = gb["codes"]
    vals = np.array([(-1 if c & 8 else 1) * mags[c & 7] for c in codes])
    want = (vals * 448.0 * np.float64(np.float32(6) / np.float32(2688))).astype(np.float32)
    np.testing.assert_array_equal(xh[0], want)


# ------------------------------------------------- second encoder (numpy)

E2M1_MAG = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def nearest_even(a64, table):
    d = np.abs(a64[..., None] - table)
    dmin = d.min(-1, keepdims=True)
    cand = d == dmin
    idx = np.arange(table.size)
    even = cand & (idx % 2 == 0)
    return np.where(even.any(-1), np.argmax(even, -1), np.argmax(cand, -1))


def e4m3_values():
    v = torch.arange(127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    return v.to(torch.float32).numpy().astype(np.float64)


def second_rowwise(xf: np.ndarray, amax: np.ndarray):
    """Rowwise cast of float32 rows xf [M, K] with per-row amax, written with
    numpy array operations and nearest-value searches."""
    M, K = xf.shape
    f32 = np.float32
    with np.errstate(divide="ignore", over="ignore"):
        senc = np.where(amax == 0, f32(1), np.minimum(f32(2688) / amax, FLT_MAX)).astype(f32)
    blk = xf.reshape(M, K // 16, 16)
    bmax = np.abs(blk).max(-1)
    s32 = ((bmax / f32(6)).astype(f32) * senc[:, None]).astype(f32)
    tab = e4m3_values()
    s8 = nearest_even(s32.astype(np.float64), tab).astype(np.uint8)
    s8v = tab[s8].astype(f32)
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        enc = np.where(s8 == 0, f32(0), np.minimum(senc[:, None] / s8v, FLT_MAX)).astype(f32)
    y = (blk * enc[..., None]).astype(f32)
    mag = nearest_even(np.abs(y).astype(np.float64), E2M1_MAG).astype(np.uint8)
    codes = mag | np.where(np.signbit(y), 8, 0).astype(np.uint8)
    codes = codes.reshape(M, K)
    data = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return data, s8.reshape(M, K // 16), (amax / f32(2688)).astype(f32)


@pytest.mark.parametrize("seed,K,splits,dist", [
    (11, 16, [16], "normal"), (12, 32, [16, 0, 32], "wide"), (13, 64, [48, 16], "heavy"),
    (14, 48, [0, 0, 16], "normal"), (15, 128, [32, 64, 0, 32], "wide")])
def test_second_encoder_agrees_on_tiny_inputs(seed, K, splits, dist):
    w = workloads.random_case(seed, K, splits, dist=dist)
    x = workloads.bits(w.x)
    xf = oracle.bf16_to_f32(x).reshape(x.shape)
    ra, ca = oracle.group_amax(x, splits)
    # brute-force amax
    np.testing.assert_array_equal(ra, np.abs(xf).max(axis=1) if K else ra)
    offs = workloads.row_offsets(splits)
    for g, m in enumerate(splits):
        want = np.abs(xf[offs[g]:offs[g] + m]).max(axis=0) if m else np.zeros(K, np.float32)
        np.testing.assert_array_equal(ca[g * K:(g + 1) * K], want)
    out = oracle.group_cast(x, splits, ra, ca)
    d, s, s2 = second_rowwise(xf, ra)
    np.testing.assert_array_equal(out["row_data"], d)
    np.testing.assert_array_equal(out["row_scale"], s)
    np.testing.assert_array_equal(out["row_s2"], s2)
    # colwise: group g's slice is the rowwise cast of the group's transpose
    for g, m in enumerate(splits):
        if m == 0:
            continue
        xt = np.ascontiguousarray(xf[offs[g]:offs[g] + m].T)
        d, s, s2 = second_rowwise(xt, ca[g * K:(g + 1) * K])
        np.testing.assert_array_equal(oracle.col_slice(out["col_data"], splits, K, g, 2), d)
        np.testing.assert_array_equal(oracle.col_slice(out["col_scale"], splits, K, g, 16), s)
        np.testing.assert_array_equal(out["col_s2"][g * K:(g + 1) * K], s2)


# -------------------------------------------------------------- invariants

def decode_all(data, scale, s2, rows, cols):
    return oracle.dequantize(data, scale, s2, rows, cols)


def check_invariants(xf, data, scale, s2, amax):
    """xf [R, C] float32 input rows, their cast (data/scale/s2) and governing
    amax per row."""
    R, C = xf.shape
    xh = decode_all(data, scale, s2, R, C)
    # (i) |x_hat| <= a (1 + 2^-22)
    bound = amax.astype(np.float64)[:, None] * (1 + 2.0 ** -22)
    assert np.all(np.abs(xh.astype(np.float64)) <= bound)
    # (ii) error at most half an E2M1 step times the block scale
    tab = e4m3_values()
    s8v = tab[scale.astype(np.int64)]                       # [R, C/16]
    sd = s2.astype(np.float64)[:, None]
    senc = np.array([oracle.s_enc(a) for a in amax], dtype=np.float32)
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        enc = np.where(scale == 0, 0, np.minimum(senc[:, None] / s8v.astype(np.float32), FLT_MAX))
    y = np.abs(xf.reshape(R, C // 16, 16).astype(np.float64) * enc[..., None])
    step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    unit = (s8v * sd)[..., None]
    err = np.abs(xf.astype(np.float64) - xh.astype(np.float64)).reshape(R, C // 16, 16)
    normal = (s8v >= 2.0 ** -6)[..., None] & (y <= 6)
    lim = 0.5 * step * unit * (1 + 2.0 ** -20) + np.abs(xf.reshape(R, C // 16, 16)) * 2.0 ** -20
    assert np.all(err[np.broadcast_to(normal, err.shape)] <= lim[np.broadcast_to(normal, err.shape)])
    # above 6 the code saturates: the error is the overshoot times the unit
    over = (y > 6)
    lim_sat = (y - 6) * unit * (1 + 2.0 ** -20) + np.abs(xf.reshape(R, C // 16, 16)) * 2.0 ** -20
    assert np.all(err[over] <= lim_sat[over])
    # (iii) the block holding a normal amax: scale 0x7E and code +-7
    codes = np.zeros((R, C), dtype=np.uint8)
    codes[:, 0::2] = data & 0xF
    codes[:, 1::2] = data >> 4
    for r in range(R):
        a = amax[r]
        if a < 1e-30:
            continue
        j = int(np.argmax(np.abs(xf[r])))
        if np.abs(xf[r, j]) != a:
            continue
        assert scale[r, j // 16] == 0x7E, (r, j)
        assert codes[r, j] & 7 == 7, (r, j, codes[r, j])
    return xh


@pytest.mark.parametrize("dist", ["normal", "wide", "heavy"])
def test_invariants_rowwise_and_colwise(dist):
    splits = [64, 0, 128, 32]
    K = 256
    w = workloads.random_case(21, K, splits, dist=dist)
    x = workloads.bits(w.x)
    xf = oracle.bf16_to_f32(x).reshape(x.shape)
    ra, ca = oracle.group_amax(x, splits)
    out = oracle.group_cast(x, splits, ra, ca)
    check_invariants(xf, out["row_data"], out["row_scale"], out["row_s2"], ra)
    offs = workloads.row_offsets(splits)
    for g, m in enumerate(splits):
        if m == 0:
            continue
        xt = np.ascontiguousarray(xf[offs[g]:offs[g] + m].T)
        check_invariants(xt, oracle.col_slice(out["col_data"], splits, K, g, 2),
                         oracle.col_slice(out["col_scale"], splits, K, g, 16),
                         out["col_s2"][g * K:(g + 1) * K], ca[g * K:(g + 1) * K])


def test_zero_rows_and_empty_groups():
    K = 64
    splits = [0, 32, 0, 16, 0]
    xf = np.zeros((48, K), dtype=np.float32)
    xf[5] = -0.0
    xf[40, 3] = 2.5  # the only non-zero element, in group 3
    x = to_bits(xf)
    ra, ca = oracle.group_amax(x, splits)
    assert np.all(ra[:40] == 0) and ra[40] == 2.5
    assert np.all(ca[:3 * K] == 0) and ca[3 * K + 3] == 2.5 and np.all(ca[4 * K:] == 0)
    out = oracle.group_cast(x, splits, ra, ca)
    z = np.ones(48, bool)
    z[40] = False
    assert np.all(out["row_scale"][z] == 0)
    assert np.all(out["row_s2"][z] == 0)
    rd = out["row_data"]
    assert np.all(rd[5] == 0x88)                    # -0 keeps its sign
    assert np.all(rd[z][np.arange(47) != 5] == 0)
    assert np.all(out["col_s2"][:3 * K] == 0) and np.all(out["col_s2"][4 * K:] == 0)
    assert out["col_data"].size == 48 * K // 2     # empty groups own no bytes


def test_oracle_rejects_bad_input():
    x = np.zeros((32, 16), dtype=np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.group_amax(x, [16, 8])               # splits do not sum to rows
    with pytest.raises(oracle.OracleError):
        oracle.group_amax(np.zeros((4, 24), np.uint16), [4])  # K % 16 != 0
    with pytest.raises(oracle.OracleError):
        oracle.group_cast(x, [24, 8], np.zeros(32, np.float32), np.zeros(32, np.float32))
    bad = x.copy()
    bad[3, 3] = 0x7F80                               # +Inf
    with pytest.raises(oracle.OracleError):
        oracle.group_amax(bad, [32])
    # an empty problem is fine
    ra, ca = oracle.group_amax(np.zeros((0, 16), np.uint16), [0, 0])
    assert ra.size == 0 and np.all(ca == 0)


def test_block_whose_scale_rounds_to_zero_encodes_signed_zeros():
    """A block far below its row's amax gets block scale 0; its element scale
    is then 0 and every element becomes +-0 (codes 0x0 / 0x8)."""
    K = 32
    xf = np.zeros((1, K), dtype=np.float32)
    xf[0, 0] = 1.0
    xf[0, 16:20] = [1e-7, -1e-7, 3e-8, -0.0]
    x = to_bits(xf)
    ra, _ = oracle.group_amax(x, [1], cols=False)
    out = oracle.group_cast(x, [1], ra, None, cols=False)
    assert out["row_scale"][0, 1] == 0
    assert out["row_data"][0, 8:].tobytes().hex() == "8080000000000000"
