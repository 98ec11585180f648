"""Python access to the plain C oracle of the grouped row-scaled NVFP4 cast.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product library
(``nvfp4_row_scaled_b200``) never does, and this package never imports it.

Every function here marshals numpy arrays into ``libnvfp4_oracle.so`` (built
from ``nvfp4_oracle.c`` on first use) and returns numpy arrays. The arithmetic
and the readings it follows are documented in ``nvfp4_oracle.c``; the pages it
cites are TransformerEngine #3649 ("single-launch grouped row-scaled NVFP4
cast", Description), #2931 ("Implement per-token NVFP4 fprop recipe",
Changes and sequence diagram), #3324 (row-scaled backward for GroupedLinear,
summary) and #3824 ("What this changes", item 2).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from .build import build_oracle

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_i64p = ctypes.POINTER(ctypes.c_int64)


def load(path: str):
    """Open an oracle library at ``path`` and declare its signatures."""
    L = ctypes.CDLL(path)
    _declare(L)
    return L


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        _lib = load(build_oracle())
    return _lib


def _declare(L):
    """Declare the C signatures of an oracle library."""
    L.nvo_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.nvo_bf16_to_f32.restype = ctypes.c_float
    L.nvo_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.nvo_e2m1_decode.restype = ctypes.c_float
    L.nvo_e2m1_encode.argtypes = [ctypes.c_float]
    L.nvo_e2m1_encode.restype = ctypes.c_uint8
    L.nvo_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.nvo_e4m3_decode.restype = ctypes.c_float
    L.nvo_e4m3_encode.argtypes = [ctypes.c_float]
    L.nvo_e4m3_encode.restype = ctypes.c_uint8
    L.nvo_e2m1_encode_array.argtypes = [_f32p, ctypes.c_int64, _u8p]
    L.nvo_e2m1_encode_array.restype = None
    L.nvo_e4m3_encode_array.argtypes = [_f32p, ctypes.c_int64, _u8p]
    L.nvo_e4m3_encode_array.restype = None
    L.nvo_s_enc.argtypes = [ctypes.c_float]
    L.nvo_s_enc.restype = ctypes.c_float
    L.nvo_s_dec.argtypes = [ctypes.c_float]
    L.nvo_s_dec.restype = ctypes.c_float
    L.nvo_block_encode.argtypes = [_f32p, ctypes.c_float, _u8p, _u8p]
    L.nvo_block_encode.restype = None
    L.nvo_group_amax.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, _i64p,
                                 ctypes.c_int32, _f32p, _f32p]
    L.nvo_group_amax.restype = ctypes.c_int
    L.nvo_group_cast.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, _i64p,
                                 ctypes.c_int32, _f32p, _f32p,
                                 _u8p, _u8p, _f32p, _u8p, _u8p, _f32p]
    L.nvo_group_cast.restype = ctypes.c_int
    L.nvo_dequantize.argtypes = [_u8p, _u8p, _f32p, ctypes.c_int64, ctypes.c_int64, _f32p]
    L.nvo_dequantize.restype = ctypes.c_int
    L.nvo_e8m0_decode.argtypes = [ctypes.c_uint8]
    L.nvo_e8m0_decode.restype = ctypes.c_float
    L.nvo_mx_block_encode.argtypes = [_f32p, _u8p, _u8p]
    L.nvo_mx_block_encode.restype = None
    L.nvo_mx_group_cast.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, _i64p, ctypes.c_int32,
                                    _u8p, _u8p, _u8p, _u8p]
    L.nvo_mx_group_cast.restype = ctypes.c_int
    L.nvo_mx_dequantize.argtypes = [_u8p, _u8p, ctypes.c_int64, ctypes.c_int64, _f32p]
    L.nvo_mx_dequantize.restype = ctypes.c_int
    L.nvo_swizzle_scales_128x4.argtypes = [_u8p, ctypes.c_int64, ctypes.c_int64, _u8p]
    L.nvo_swizzle_scales_128x4.restype = ctypes.c_int
    L.nvo_f32_to_bf16.argtypes = [ctypes.c_float]
    L.nvo_f32_to_bf16.restype = ctypes.c_uint16
    L.nvo_row_post_scale.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, _f32p, _f32p, _f32p, _u16p]
    L.nvo_row_post_scale.restype = ctypes.c_int


class OracleError(RuntimeError):
    pass


def _ptr(a: Optional[np.ndarray], t):
    if a is None:
        return ctypes.cast(None, t)
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: oracle error {rc} "
                          f"({'bad argument' if rc == 1 else 'non-finite input'})")


def _splits(m_splits: Sequence[int]) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(list(m_splits), dtype=np.int64))


def _x(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns as a C-contiguous uint16 array [sum_M, K]."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return x


# ------------------------------------------------------------------ formats

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def e2m1_decode(code: int) -> float:
    return float(lib().nvo_e2m1_decode(code))


def e4m3_decode(code: int) -> float:
    return float(lib().nvo_e4m3_decode(code))


def e2m1_encode(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    lib().nvo_e2m1_encode_array(_ptr(y, _f32p), y.size, _ptr(out, _u8p))
    return out


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().nvo_e4m3_encode_array(_ptr(v, _f32p), v.size, _ptr(out, _u8p))
    return out


def s_enc(a: float) -> np.float32:
    return np.float32(lib().nvo_s_enc(np.float32(a)))


def s_dec(a: float) -> np.float32:
    return np.float32(lib().nvo_s_dec(np.float32(a)))


def block_encode(x16: np.ndarray, senc: float):
    """One 16-element block -> (scale byte, 16 element codes)."""
    x16 = np.ascontiguousarray(x16, dtype=np.float32)
    assert x16.size == 16
    s8 = np.zeros(1, dtype=np.uint8)
    codes = np.zeros(16, dtype=np.uint8)
    lib().nvo_block_encode(_ptr(x16, _f32p), np.float32(senc), _ptr(s8, _u8p), _ptr(codes, _u8p))
    return int(s8[0]), codes


# ------------------------------------------------------------ grouped path

def group_amax(x: np.ndarray, m_splits: Sequence[int], rows: bool = True, cols: bool = True):
    """Grouped amax of bf16 bits x [sum_M, K] -> (row_amax [sum_M], col_amax [E*K])."""
    x = _x(x)
    sum_M, K = x.shape
    ms = _splits(m_splits)
    E = len(ms)
    row = np.zeros(sum_M, dtype=np.float32) if rows else None
    col = np.zeros(E * K, dtype=np.float32) if cols else None
    rc = lib().nvo_group_amax(_ptr(x, _u16p), sum_M, K, _ptr(ms, _i64p), E,
                              _ptr(row, _f32p), _ptr(col, _f32p))
    _check(rc, "group_amax")
    return row, col


def group_cast(x: np.ndarray, m_splits: Sequence[int], row_amax: Optional[np.ndarray],
               col_amax: Optional[np.ndarray], rows: bool = True, cols: bool = True) -> dict:
    """Grouped cast. Returns a dict with row_data [sum_M, K/2], row_scale
    [sum_M, K/16], row_s2 [sum_M], col_data [sum_M*K/2] (per-group transposed
    slices, flat), col_scale [sum_M*K/16] (flat), col_s2 [E*K]."""
    x = _x(x)
    sum_M, K = x.shape
    ms = _splits(m_splits)
    E = len(ms)
    out = {}
    if rows:
        out["row_data"] = np.zeros((sum_M, K // 2), dtype=np.uint8)
        out["row_scale"] = np.zeros((sum_M, K // 16), dtype=np.uint8)
        out["row_s2"] = np.zeros(sum_M, dtype=np.float32)
        row_amax = np.ascontiguousarray(row_amax, dtype=np.float32)
    if cols:
        out["col_data"] = np.zeros(sum_M * K // 2, dtype=np.uint8)
        out["col_scale"] = np.zeros(sum_M * K // 16, dtype=np.uint8)
        out["col_s2"] = np.zeros(E * K, dtype=np.float32)
        col_amax = np.ascontiguousarray(col_amax, dtype=np.float32)
    rc = lib().nvo_group_cast(
        _ptr(x, _u16p), sum_M, K, _ptr(ms, _i64p), E,
        _ptr(row_amax if rows else None, _f32p), _ptr(col_amax if cols else None, _f32p),
        _ptr(out.get("row_data"), _u8p), _ptr(out.get("row_scale"), _u8p),
        _ptr(out.get("row_s2"), _f32p),
        _ptr(out.get("col_data"), _u8p), _ptr(out.get("col_scale"), _u8p),
        _ptr(out.get("col_s2"), _f32p))
    _check(rc, "group_cast")
    return out


def dequantize(data: np.ndarray, scale: np.ndarray, s2: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Decode [rows, cols] from packed codes [rows, cols/2], E4M3 scales
    [rows, cols/16] and one decode scale per row."""
    data = np.ascontiguousarray(data, dtype=np.uint8).reshape(-1)
    scale = np.ascontiguousarray(scale, dtype=np.uint8).reshape(-1)
    s2 = np.ascontiguousarray(s2, dtype=np.float32).reshape(-1)
    out = np.zeros((rows, cols), dtype=np.float32)
    rc = lib().nvo_dequantize(_ptr(data, _u8p), _ptr(scale, _u8p), _ptr(s2, _f32p),
                              rows, cols, _ptr(out, _f32p))
    _check(rc, "dequantize")
    return out


def col_slice(col_flat: np.ndarray, m_splits: Sequence[int], K: int, g: int, per_elem: int) -> np.ndarray:
    """View group g's transposed slice [K, m_g/per_elem] of a flat colwise
    buffer (per_elem = 2 for data, 16 for scales)."""
    ms = list(m_splits)
    o = sum(ms[:g])
    m = ms[g]
    start = K * o // per_elem
    return col_flat[start:start + K * m // per_elem].reshape(K, m // per_elem)


# --------------------------------------------------- consumer side of the cast

def swizzle_scales_128x4(scale: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """The 128x4-tiled layout of a scale matrix [rows, cols] (flat uint8,
    ceil(rows/128)*128 * ceil(cols/4)*4 bytes)."""
    scale = np.ascontiguousarray(scale, dtype=np.uint8).reshape(-1)
    assert scale.size == rows * cols
    out = np.zeros(((rows + 127) // 128) * 128 * ((cols + 3) // 4) * 4, dtype=np.uint8)
    _check(lib().nvo_swizzle_scales_128x4(_ptr(scale, _u8p), rows, cols, _ptr(out, _u8p)),
           "swizzle_scales_128x4")
    return out


def f32_to_bf16(v: float) -> int:
    return int(lib().nvo_f32_to_bf16(float(v)))


def row_post_scale(x: np.ndarray, amax: np.ndarray, bias: Optional[np.ndarray] = None):
    """(f32 [rows, cols], bf16 bits [rows, cols]) of the per-row post-scale."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    amax = np.ascontiguousarray(amax, dtype=np.float32).reshape(-1)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32).reshape(-1)
    of = np.zeros((rows, cols), dtype=np.float32)
    ob = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().nvo_row_post_scale(_ptr(x, _f32p), rows, cols, _ptr(amax, _f32p), _ptr(b, _f32p),
                                    _ptr(of, _f32p), _ptr(ob, _u16p)), "row_post_scale")
    return of, ob


def swizzle_cast_scales(out: dict, m_splits: Sequence[int], K: int) -> dict:
    """The scale outputs of a grouped cast in the 128x4-tiled layout: rowwise
    [sum_M, K/16] as one matrix, colwise per group [K, m_g/16] at its own
    offset K*o_g/16 (groups must be multiples of 128 rows)."""
    res = {}
    if "row_scale" in out:
        rs = np.asarray(out["row_scale"]).reshape(-1)
        rows = rs.size // (K // 16)
        res["row_scale"] = swizzle_scales_128x4(rs, rows, K // 16)
    if "col_scale" in out:
        cs = np.asarray(out["col_scale"]).reshape(-1)
        parts = []
        for g, m in enumerate(m_splits):
            if m:
                parts.append(swizzle_scales_128x4(col_slice(cs, m_splits, K, g, 16), K, m // 16))
        res["col_scale"] = np.concatenate(parts) if parts else np.zeros(0, np.uint8)
    return res


# -------------------------------------------------------------------- MXFP4

def e8m0_decode(code: int) -> float:
    return float(lib().nvo_e8m0_decode(int(code)))


def mx_block_encode(x32: np.ndarray):
    """(E8M0 scale byte, 32 codes) of one MXFP4 block."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    assert x32.size == 32
    s8 = np.zeros(1, dtype=np.uint8)
    codes = np.zeros(32, dtype=np.uint8)
    lib().nvo_mx_block_encode(_ptr(x32, _f32p), _ptr(s8, _u8p), _ptr(codes, _u8p))
    return int(s8[0]), codes


def mx_group_cast(x: np.ndarray, m_splits: Sequence[int], rows: bool = True, cols: bool = True) -> dict:
    """Grouped MXFP4 cast of bf16 bits x [sum_M, K]: row_data [sum_M, K/2],
    row_scale [sum_M, K/32], col_data / col_scale flat (group g at K*o_g/2,
    K*o_g/32, shapes [K, m_g/2], [K, m_g/32])."""
    x = _x(x)
    M, K = x.shape
    sp = _splits(m_splits)
    out = {}
    if rows:
        out["row_data"] = np.zeros((M, K // 2), dtype=np.uint8)
        out["row_scale"] = np.zeros((M, K // 32), dtype=np.uint8)
    if cols:
        out["col_data"] = np.zeros(M * K // 2, dtype=np.uint8)
        out["col_scale"] = np.zeros(M * K // 32, dtype=np.uint8)
    rc = lib().nvo_mx_group_cast(_ptr(x, _u16p), M, K, _ptr(sp, _i64p), len(sp),
                                 _ptr(out.get("row_data"), _u8p), _ptr(out.get("row_scale"), _u8p),
                                 _ptr(out.get("col_data"), _u8p), _ptr(out.get("col_scale"), _u8p))
    _check(rc, "mx_group_cast")
    return out


def mx_dequantize(data: np.ndarray, scale: np.ndarray, rows: int, cols: int) -> np.ndarray:
    data = np.ascontiguousarray(data, dtype=np.uint8).reshape(-1)
    scale = np.ascontiguousarray(scale, dtype=np.uint8).reshape(-1)
    out = np.zeros((rows, cols), dtype=np.float32)
    _check(lib().nvo_mx_dequantize(_ptr(data, _u8p), _ptr(scale, _u8p), rows, cols, _ptr(out, _f32p)),
           "mx_dequantize")
    return out
