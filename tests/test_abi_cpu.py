"""The C-ABI library, checked without a GPU.

- it builds (nvcc cross-compiles sm_100a here) and loads;
- it exports every function that include/*.h declares;
- host-side argument checks return their status before anything is enqueued
  (none of these calls reaches the CUDA runtime).
"""
import ctypes
import glob
import os
import re

import pytest

from nvfp4_row_scaled_b200 import abi
from nvfp4_row_scaled_b200.build import build_library

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_library()
    return abi.lib()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(nvfp4_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("nvfp4_group_amax", "nvfp4_group_cast", "nvfp4_group_amax_graphsafe",
                 "nvfp4_group_cast_graphsafe", "nvfp4_dequantize", "nvfp4_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {abi.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(declared_functions()), exported ^ set(declared_functions())


def test_status_strings(L):
    for code, name in [(0, "NVFP4_OK"), (1, "NVFP4_ERR_INVALID_ARG"), (2, "NVFP4_ERR_UNSUPPORTED"),
                       (3, "NVFP4_ERR_CUDA"), (4, "NVFP4_ERR_ROUTING")]:
        assert abi.status_name(code) == name


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every case fails its host checks first


def amax(L, x, sum_M, K, splits, row=FAKE, col=FAKE):
    arr = (ctypes.c_int64 * max(len(splits), 1))(*splits) if splits is not None else None
    return L.nvfp4_group_amax(x, sum_M, K, arr, len(splits or []), row, col, None)


@pytest.mark.parametrize("sum_M,K,splits,want", [
    (256, 24, [256], abi.NVFP4_ERR_INVALID_ARG),       # K % 16
    (256, 128, [128, 64], abi.NVFP4_ERR_INVALID_ARG),  # splits do not add up
    (256, 128, [384, -128], abi.NVFP4_ERR_INVALID_ARG),  # negative split
    (192, 128, [56, 136], abi.NVFP4_ERR_UNSUPPORTED),  # group not a multiple of 16
    (-1, 128, [], abi.NVFP4_ERR_INVALID_ARG),
])
def test_amax_host_checks(L, sum_M, K, splits, want):
    assert amax(L, FAKE, sum_M, K, splits) == want


def test_amax_pointer_checks(L):
    assert amax(L, None, 128, 128, [128]) == abi.NVFP4_ERR_INVALID_ARG
    assert amax(L, ctypes.c_void_p(0x10008), 128, 128, [128]) == abi.NVFP4_ERR_UNSUPPORTED
    assert amax(L, FAKE, 128, 128, [128], row=None, col=None) == abi.NVFP4_ERR_INVALID_ARG
    assert amax(L, FAKE, 128, 128, [128] * (abi.NVFP4_MAX_GROUPS + 1)) == abi.NVFP4_ERR_UNSUPPORTED


def test_cast_output_descriptor_checks(L):
    arr = (ctypes.c_int64 * 1)(128)
    o = abi.Outputs(row_data=0x10000, row_scale=None, row_s2=0x10000)  # partial direction
    assert L.nvfp4_group_cast(FAKE, 128, 128, arr, 1, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_INVALID_ARG
    o = abi.Outputs(row_data=0x10004, row_scale=0x10000, row_s2=0x10000)  # misaligned data
    assert L.nvfp4_group_cast(FAKE, 128, 128, arr, 1, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_UNSUPPORTED
    o = abi.Outputs(row_data=0x10000, row_scale=0x10000, row_s2=0x10000)
    assert L.nvfp4_group_cast(FAKE, 128, 128, arr, 1, None, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_INVALID_ARG  # row direction without row_amax
    assert L.nvfp4_group_cast(FAKE, 128, 128, arr, 1, FAKE, FAKE, None, None) == \
        abi.NVFP4_ERR_INVALID_ARG


def test_graphsafe_host_checks(L):
    f = L.nvfp4_group_amax_graphsafe
    assert f(FAKE, 256, 128, FAKE, FAKE, 2, FAKE, FAKE, None, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 256, 128, FAKE, None, 2, FAKE, FAKE, FAKE, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 256, 120, FAKE, FAKE, 2, FAKE, FAKE, FAKE, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 256, 128, ctypes.c_void_p(0x10004), FAKE, 2, FAKE, FAKE, FAKE, None) == \
        abi.NVFP4_ERR_UNSUPPORTED


def test_quantize_workspace_bytes(L):
    f = abi.nvfp4_group_quantize_workspace_bytes
    # 64 header words, then one done counter per group, rounded up to 64 words,
    # then one word per row (graph-safe)
    assert f(0, 0) == 4 * 64
    assert f(0, 1) == 4 * 128
    assert f(0, 64) == 4 * 128
    assert f(0, 65) == 4 * 192
    assert f(0, abi.NVFP4_MAX_GROUPS) == 4352
    assert f(1000, 256) == 4 * (320 + 1000)
    assert f(-1, 4) == 0 and f(0, -1) == 0 and f(0, abi.NVFP4_MAX_GROUPS + 1) == 0


def test_quantize_host_checks(L):
    arr = (ctypes.c_int64 * 2)(128, 128)
    o = abi.Outputs(row_data=0x10000, row_scale=0x10000, row_s2=0x10000,
                    col_data=0x10000, col_scale=0x10000, col_s2=0x10000)
    need = abi.nvfp4_group_quantize_workspace_bytes(0, 2)
    q = L.nvfp4_group_quantize

    def call(ws=FAKE, nbytes=need, row=FAKE, col=FAKE, K=128, out=o):
        return q(FAKE, 256, K, arr, 2, row, col, ctypes.byref(out) if out is not None else None,
                 ws, nbytes, None)
    assert call(ws=None) == abi.NVFP4_ERR_INVALID_ARG
    assert call(nbytes=need - 4) == abi.NVFP4_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(0x10004)) == abi.NVFP4_ERR_UNSUPPORTED
    assert call(row=None) == abi.NVFP4_ERR_INVALID_ARG     # rows requested, no row_amax
    assert call(col=None) == abi.NVFP4_ERR_INVALID_ARG     # columns requested, no col_amax
    assert call(K=120) == abi.NVFP4_ERR_INVALID_ARG
    assert call(out=None) == abi.NVFP4_ERR_INVALID_ARG
    g = L.nvfp4_group_quantize_graphsafe
    small = abi.nvfp4_group_quantize_workspace_bytes(256, 2) - 4
    assert g(FAKE, 256, 128, FAKE, FAKE, 2, FAKE, FAKE, ctypes.byref(o), FAKE, small, FAKE, None) == \
        abi.NVFP4_ERR_INVALID_ARG  # the graph-safe call needs the row accumulators too
    assert g(FAKE, 256, 128, FAKE, FAKE, 2, FAKE, FAKE, ctypes.byref(o), FAKE, small + 4, None, None) == \
        abi.NVFP4_ERR_INVALID_ARG  # no status word


def test_quantize_noalloc_host_checks(L):
    arr = (ctypes.c_int64 * 2)(128, 128)
    o = abi.Outputs(row_data=0x10000, row_scale=0x10000, row_s2=0x10000,
                    col_data=0x10000, col_scale=0x10000, col_s2=0x10000)
    f = L.nvfp4_group_quantize_noalloc
    assert f(FAKE, 256, 120, arr, 2, FAKE, FAKE, ctypes.byref(o), None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 256, 128, arr, 2, None, FAKE, ctypes.byref(o), None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 256, 128, arr, 2, ctypes.c_void_p(0x10004), FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_UNSUPPORTED  # the amax vectors are copied in 512-byte runs
    big = (ctypes.c_int64 * (abi.NVFP4_MAX_GROUPS + 1))()
    big[0] = 256
    assert f(FAKE, 256, 128, big, abi.NVFP4_MAX_GROUPS + 1, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_UNSUPPORTED  # beyond the static scratch


def test_post_scale_host_checks(L):
    f = L.nvfp4_row_post_scale
    assert f(FAKE, 4, 6, FAKE, None, FAKE, abi.NVFP4_OUT_F32, None) == abi.NVFP4_ERR_UNSUPPORTED  # cols % 4
    assert f(FAKE, 4, 8, FAKE, None, FAKE, 7, None) == abi.NVFP4_ERR_INVALID_ARG  # unknown dtype
    assert f(None, 4, 8, FAKE, None, FAKE, abi.NVFP4_OUT_F32, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, 4, 8, FAKE, None, ctypes.c_void_p(0x10008), abi.NVFP4_OUT_F32, None) == \
        abi.NVFP4_ERR_UNSUPPORTED  # f32 output must be 16-byte aligned
    assert f(FAKE, 0, 8, FAKE, None, FAKE, abi.NVFP4_OUT_BF16, None) == abi.NVFP4_OK  # empty


def test_scale_layout_must_be_known(L):
    arr = (ctypes.c_int64 * 1)(128)
    o = abi.Outputs(row_data=0x10000, row_scale=0x10000, row_s2=0x10000, scale_layout=5)
    assert L.nvfp4_group_cast(FAKE, 128, 128, arr, 1, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_INVALID_ARG


def test_mx_host_checks(L):
    arr = (ctypes.c_int64 * 2)(128, 128)
    o = abi.MxOutputs(row_data=0x10000, row_scale=None)  # partial direction
    assert L.nvfp4_mx_group_cast(FAKE, 256, 128, arr, 2, ctypes.byref(o), None) == abi.NVFP4_ERR_INVALID_ARG
    o = abi.MxOutputs(row_data=0x10000, row_scale=0x10000)
    # K must be a multiple of the 32-element block, as in the oracle
    assert L.nvfp4_mx_group_cast(FAKE, 256, 144, arr, 2, ctypes.byref(o), None) == abi.NVFP4_ERR_INVALID_ARG
    # groups must be multiples of 32 rows (a colwise block lies in one group)
    arr2 = (ctypes.c_int64 * 2)(48, 208)
    assert L.nvfp4_mx_group_cast(FAKE, 256, 160, arr2, 2, ctypes.byref(o), None) == abi.NVFP4_ERR_UNSUPPORTED
    f = L.nvfp4_mx_dequantize
    assert f(FAKE, FAKE, 4, 48, FAKE, None) == abi.NVFP4_ERR_INVALID_ARG  # cols % 32
    assert f(FAKE, FAKE, 4, 64, ctypes.c_void_p(0x10008), None) == abi.NVFP4_ERR_UNSUPPORTED


def test_dequantize_host_checks(L):
    f = L.nvfp4_dequantize
    assert f(FAKE, FAKE, FAKE, 4, 24, FAKE, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, -1, 16, FAKE, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(None, FAKE, FAKE, 4, 16, FAKE, None) == abi.NVFP4_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 4, 16, ctypes.c_void_p(0x10008), None) == abi.NVFP4_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 0, 16, FAKE, None) == abi.NVFP4_OK  # empty: nothing to do


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(abi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(abi, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        abi.lib()


def test_k_multiple_of_128_only_where_needed(L):
    """The two-step calls take any K % 16 == 0, and so do the host-split
    one-launch calls (other routings run as the two launches); the
    graph-safe one-launch call and the tiled-scale layout need K % 128 == 0
    and refuse other K up front, before anything is enqueued."""
    arr = (ctypes.c_int64 * 1)(256)
    o = abi.Outputs(row_data=0x10000, row_scale=0x10000, row_s2=0x10000,
                    col_data=0x10000, col_scale=0x10000, col_s2=0x10000)
    ws = abi.nvfp4_group_quantize_workspace_bytes(256, 1)
    assert L.nvfp4_group_quantize_graphsafe(FAKE, 256, 144, FAKE, FAKE, 1, FAKE, FAKE, ctypes.byref(o), FAKE,
                                            ws, FAKE, None) == abi.NVFP4_ERR_UNSUPPORTED
    o.scale_layout = abi.NVFP4_SCALE_TILED_128X4
    assert L.nvfp4_group_quantize(FAKE, 256, 144, arr, 1, FAKE, FAKE, ctypes.byref(o), FAKE, ws, None) == \
        abi.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_group_quantize_noalloc(FAKE, 256, 144, arr, 1, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_group_cast(FAKE, 256, 144, arr, 1, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_group_cast_graphsafe(FAKE, 256, 144, FAKE, FAKE, 1, FAKE, FAKE, ctypes.byref(o), FAKE,
                                        None) == abi.NVFP4_ERR_UNSUPPORTED
    # 128-row groups are needed by the tiled layout in every call
    arr2 = (ctypes.c_int64 * 2)(48, 208)
    assert L.nvfp4_group_quantize(FAKE, 256, 128, arr2, 2, FAKE, FAKE, ctypes.byref(o), FAKE, ws, None) == \
        abi.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_group_cast(FAKE, 256, 128, arr2, 2, FAKE, FAKE, ctypes.byref(o), None) == \
        abi.NVFP4_ERR_UNSUPPORTED