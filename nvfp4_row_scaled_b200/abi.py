"""Thin ctypes binding of ``libnvfp4rs.so`` (declared in ``include/nvfp4rs.h``).

Argument marshalling only: every function here checks that tensors are CUDA,
contiguous and of the right dtype, turns them into device pointers, passes the
current torch stream, and raises ``NVFP4Error`` on a non-OK status. All of the
method's work happens in the library's kernels. If the library is not built,
every call raises; there is no fallback.

Names follow the C entry points. Tensors:
  x            bf16 [rows, K]
  row_amax     fp32 [rows]          col_amax  fp32 [E*K]
  row_data     uint8 [rows, K/2]    row_scale uint8 [rows, K/16]   row_s2 fp32 [rows]
  col_data     uint8 [rows*K/2]     col_scale uint8 [rows*K/16]    col_s2 fp32 [E*K]
(colwise buffers hold each group's transposed [K, m_g/2] / [K, m_g/16] slice
at byte offsets K*o_g/2 and K*o_g/16).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# NVFP4RS_LIBRARY names another build of the same library to load instead
# (the bounds-checked debug build, libnvfp4rs_debug.so, for instance)
LIB_PATH = os.environ.get("NVFP4RS_LIBRARY") or os.path.join(HERE, "libnvfp4rs.so")

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_UNSUPPORTED = 2
NVFP4_ERR_CUDA = 3
NVFP4_ERR_ROUTING = 4
NVFP4_ERR_TIMEOUT = 5
NVFP4_MAX_GROUPS = 1024
NVFP4_SCALE_COMPACT = 0
NVFP4_SCALE_TILED_128X4 = 1
NVFP4_OUT_F32 = 0
NVFP4_OUT_BF16 = 1

_lib = None


class NVFP4Error(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_name(status)} ({status})")
        self.status = status


class Outputs(ctypes.Structure):
    """Mirror of ``nvfp4_outputs``."""
    _fields_ = [("row_data", ctypes.c_void_p), ("row_scale", ctypes.c_void_p),
                ("row_s2", ctypes.c_void_p), ("col_data", ctypes.c_void_p),
                ("col_scale", ctypes.c_void_p), ("col_s2", ctypes.c_void_p),
                ("scale_layout", ctypes.c_int32)]


class MxOutputs(ctypes.Structure):
    """Mirror of ``nvfp4_mx_outputs``."""
    _fields_ = [("row_data", ctypes.c_void_p), ("row_scale", ctypes.c_void_p),
                ("col_data", ctypes.c_void_p), ("col_scale", ctypes.c_void_p)]


def lib():
    """Open the library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               f"`python -m nvfp4_row_scaled_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.nvfp4_group_amax.argtypes = [vp, i64, i64, vp, i32, vp, vp, vp]
        L.nvfp4_group_cast.argtypes = [vp, i64, i64, vp, i32, vp, vp, ctypes.POINTER(Outputs), vp]
        L.nvfp4_group_amax_graphsafe.argtypes = [vp, i64, i64, vp, vp, i32, vp, vp, vp, vp]
        L.nvfp4_group_cast_graphsafe.argtypes = [vp, i64, i64, vp, vp, i32, vp, vp,
                                                 ctypes.POINTER(Outputs), vp, vp]
        L.nvfp4_dequantize.argtypes = [vp, vp, vp, i64, i64, vp, vp]
        sz = ctypes.c_size_t
        L.nvfp4_group_quantize_workspace_bytes.argtypes = [i64, i32]
        L.nvfp4_group_quantize_workspace_bytes.restype = sz
        L.nvfp4_group_quantize.argtypes = [vp, i64, i64, vp, i32, vp, vp, ctypes.POINTER(Outputs),
                                           vp, sz, vp]
        L.nvfp4_group_quantize_graphsafe.argtypes = [vp, i64, i64, vp, vp, i32, vp, vp,
                                                     ctypes.POINTER(Outputs), vp, sz, vp, vp]
        L.nvfp4_mx_group_cast.argtypes = [vp, i64, i64, vp, i32, ctypes.POINTER(MxOutputs), vp]
        L.nvfp4_mx_group_cast_graphsafe.argtypes = [vp, i64, i64, vp, vp, i32, ctypes.POINTER(MxOutputs),
                                                    vp, vp]
        L.nvfp4_mx_dequantize.argtypes = [vp, vp, i64, i64, vp, vp]
        for f in ("nvfp4_mx_group_cast", "nvfp4_mx_group_cast_graphsafe", "nvfp4_mx_dequantize"):
            getattr(L, f).restype = ctypes.c_int
        L.nvfp4_row_post_scale.argtypes = [vp, i64, i64, vp, vp, vp, i32, vp]
        L.nvfp4_row_post_scale.restype = ctypes.c_int
        L.nvfp4_group_quantize_noalloc.argtypes = [vp, i64, i64, vp, i32, vp, vp,
                                                   ctypes.POINTER(Outputs), vp]
        for f in ("nvfp4_group_amax", "nvfp4_group_cast", "nvfp4_group_amax_graphsafe",
                  "nvfp4_group_cast_graphsafe", "nvfp4_dequantize", "nvfp4_group_quantize",
                  "nvfp4_group_quantize_graphsafe", "nvfp4_group_quantize_noalloc"):
            getattr(L, f).restype = ctypes.c_int
        L.nvfp4_status_string.argtypes = [ctypes.c_int]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_name(status: int) -> str:
    return lib().nvfp4_status_string(int(status)).decode()


# ----------------------------------------------------------- marshalling

def _dev(t: Optional[torch.Tensor], dtype: torch.dtype, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _splits(m_splits: Sequence[int]):
    arr = (ctypes.c_int64 * max(len(m_splits), 1))(*[int(m) for m in m_splits])
    return arr, len(m_splits)


def _outputs(out: Dict[str, torch.Tensor], scale_layout: int = NVFP4_SCALE_COMPACT) -> Outputs:
    o = Outputs()
    o.scale_layout = int(scale_layout)
    for name, dt in (("row_data", torch.uint8), ("row_scale", torch.uint8), ("row_s2", torch.float32),
                     ("col_data", torch.uint8), ("col_scale", torch.uint8), ("col_s2", torch.float32)):
        p = _dev(out.get(name), dt, name)
        setattr(o, name, p.value if p is not None else None)
    return o


def _groups(first_dims: Optional[torch.Tensor], num_groups: Optional[int]) -> int:
    """Group count of a graph-safe call: first_dims.numel(), or num_groups for
    uniform groups (first_dims and tensor_offsets both None)."""
    if first_dims is not None:
        return first_dims.numel()
    if num_groups is None:
        raise ValueError("uniform groups (no first_dims) need num_groups")
    return int(num_groups)


def _check(rc: int, what: str):
    if rc != NVFP4_OK:
        raise NVFP4Error(what, rc)


# ------------------------------------------------------------ entry points

def nvfp4_group_amax(x: torch.Tensor, m_splits: Sequence[int], row_amax: Optional[torch.Tensor],
                     col_amax: Optional[torch.Tensor], stream=None) -> None:
    arr, E = _splits(m_splits)
    rc = lib().nvfp4_group_amax(_dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1], arr, E,
                                _dev(row_amax, torch.float32, "row_amax"),
                                _dev(col_amax, torch.float32, "col_amax"), _stream(stream))
    _check(rc, "nvfp4_group_amax")


def nvfp4_group_cast(x: torch.Tensor, m_splits: Sequence[int], row_amax: Optional[torch.Tensor],
                     col_amax: Optional[torch.Tensor], out: Dict[str, torch.Tensor],
                     stream=None, scale_layout: int = NVFP4_SCALE_COMPACT) -> None:
    arr, E = _splits(m_splits)
    o = _outputs(out, scale_layout)
    rc = lib().nvfp4_group_cast(_dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1], arr, E,
                                _dev(row_amax, torch.float32, "row_amax"),
                                _dev(col_amax, torch.float32, "col_amax"), ctypes.byref(o),
                                _stream(stream))
    _check(rc, "nvfp4_group_cast")


def nvfp4_group_amax_graphsafe(x: torch.Tensor, first_dims: torch.Tensor,
                               tensor_offsets: torch.Tensor, row_amax: Optional[torch.Tensor],
                               col_amax: Optional[torch.Tensor], status: torch.Tensor,
                               stream=None, num_groups: Optional[int] = None) -> None:
    rc = lib().nvfp4_group_amax_graphsafe(
        _dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1],
        _dev(first_dims, torch.int64, "first_dims"), _dev(tensor_offsets, torch.int64, "tensor_offsets"),
        _groups(first_dims, num_groups), _dev(row_amax, torch.float32, "row_amax"),
        _dev(col_amax, torch.float32, "col_amax"), _dev(status, torch.int32, "status"),
        _stream(stream))
    _check(rc, "nvfp4_group_amax_graphsafe")


def nvfp4_group_cast_graphsafe(x: torch.Tensor, first_dims: torch.Tensor,
                               tensor_offsets: torch.Tensor, row_amax: Optional[torch.Tensor],
                               col_amax: Optional[torch.Tensor], out: Dict[str, torch.Tensor],
                               status: torch.Tensor, stream=None,
                               scale_layout: int = NVFP4_SCALE_COMPACT,
                               num_groups: Optional[int] = None) -> None:
    o = _outputs(out, scale_layout)
    rc = lib().nvfp4_group_cast_graphsafe(
        _dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1],
        _dev(first_dims, torch.int64, "first_dims"), _dev(tensor_offsets, torch.int64, "tensor_offsets"),
        _groups(first_dims, num_groups), _dev(row_amax, torch.float32, "row_amax"),
        _dev(col_amax, torch.float32, "col_amax"), ctypes.byref(o),
        _dev(status, torch.int32, "status"), _stream(stream))
    _check(rc, "nvfp4_group_cast_graphsafe")


def nvfp4_group_quantize_workspace_bytes(capacity_rows: int, num_groups: int) -> int:
    return int(lib().nvfp4_group_quantize_workspace_bytes(int(capacity_rows), int(num_groups)))


def _workspace(ws: torch.Tensor):
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


def nvfp4_group_quantize(x: torch.Tensor, m_splits: Sequence[int], row_amax: Optional[torch.Tensor],
                         col_amax: Optional[torch.Tensor], out: Dict[str, torch.Tensor],
                         workspace: torch.Tensor, stream=None, scale_layout: int = NVFP4_SCALE_COMPACT) -> None:
    arr, E = _splits(m_splits)
    o = _outputs(out, scale_layout)
    wp, wb = _workspace(workspace)
    rc = lib().nvfp4_group_quantize(_dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1], arr, E,
                                    _dev(row_amax, torch.float32, "row_amax"),
                                    _dev(col_amax, torch.float32, "col_amax"), ctypes.byref(o),
                                    wp, wb, _stream(stream))
    _check(rc, "nvfp4_group_quantize")


def nvfp4_group_quantize_graphsafe(x: torch.Tensor, first_dims: torch.Tensor,
                                   tensor_offsets: torch.Tensor, row_amax: Optional[torch.Tensor],
                                   col_amax: Optional[torch.Tensor], out: Dict[str, torch.Tensor],
                                   workspace: torch.Tensor, status: torch.Tensor,
                                   stream=None, scale_layout: int = NVFP4_SCALE_COMPACT,
                                   num_groups: Optional[int] = None) -> None:
    o = _outputs(out, scale_layout)
    wp, wb = _workspace(workspace)
    rc = lib().nvfp4_group_quantize_graphsafe(
        _dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1],
        _dev(first_dims, torch.int64, "first_dims"), _dev(tensor_offsets, torch.int64, "tensor_offsets"),
        _groups(first_dims, num_groups), _dev(row_amax, torch.float32, "row_amax"),
        _dev(col_amax, torch.float32, "col_amax"), ctypes.byref(o), wp, wb,
        _dev(status, torch.int32, "status"), _stream(stream))
    _check(rc, "nvfp4_group_quantize_graphsafe")


def nvfp4_group_quantize_noalloc(x: torch.Tensor, m_splits: Sequence[int],
                                 row_amax: Optional[torch.Tensor], col_amax: Optional[torch.Tensor],
                                 out: Dict[str, torch.Tensor], stream=None, scale_layout: int = NVFP4_SCALE_COMPACT) -> None:
    """nvfp4_group_quantize with the library's static scratch (no workspace)."""
    arr, E = _splits(m_splits)
    o = _outputs(out, scale_layout)
    rc = lib().nvfp4_group_quantize_noalloc(_dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1], arr, E,
                                            _dev(row_amax, torch.float32, "row_amax"),
                                            _dev(col_amax, torch.float32, "col_amax"), ctypes.byref(o),
                                            _stream(stream))
    _check(rc, "nvfp4_group_quantize_noalloc")


def nvfp4_row_post_scale(gemm_out: torch.Tensor, row_amax: torch.Tensor, out: torch.Tensor,
                         bias: Optional[torch.Tensor] = None, stream=None) -> None:
    """out = gemm_out * row_amax[:, None] (+ bias), as fp32 or bf16 (out's dtype)."""
    if out.dtype == torch.float32:
        dt = NVFP4_OUT_F32
    elif out.dtype == torch.bfloat16:
        dt = NVFP4_OUT_BF16
    else:
        raise ValueError("out must be float32 or bfloat16")
    if out.shape != gemm_out.shape:
        raise ValueError("out must have gemm_out's shape")
    rows, cols = gemm_out.shape
    rc = lib().nvfp4_row_post_scale(_dev(gemm_out, torch.float32, "gemm_out"), rows, cols,
                                    _dev(row_amax, torch.float32, "row_amax"),
                                    _dev(bias, torch.float32, "bias"), _dev(out, out.dtype, "out"), dt,
                                    _stream(stream))
    _check(rc, "nvfp4_row_post_scale")


def _mx_outputs(out: Dict[str, torch.Tensor]) -> MxOutputs:
    o = MxOutputs()
    for name in ("row_data", "row_scale", "col_data", "col_scale"):
        p = _dev(out.get(name), torch.uint8, name)
        setattr(o, name, p.value if p is not None else None)
    return o


def nvfp4_mx_group_cast(x: torch.Tensor, m_splits: Sequence[int], out: Dict[str, torch.Tensor],
                        stream=None) -> None:
    arr, E = _splits(m_splits)
    o = _mx_outputs(out)
    rc = lib().nvfp4_mx_group_cast(_dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1], arr, E,
                                   ctypes.byref(o), _stream(stream))
    _check(rc, "nvfp4_mx_group_cast")


def nvfp4_mx_group_cast_graphsafe(x: torch.Tensor, first_dims: Optional[torch.Tensor],
                                  tensor_offsets: Optional[torch.Tensor], out: Dict[str, torch.Tensor],
                                  status: torch.Tensor, stream=None,
                                  num_groups: Optional[int] = None) -> None:
    o = _mx_outputs(out)
    rc = lib().nvfp4_mx_group_cast_graphsafe(
        _dev(x, torch.bfloat16, "x"), x.shape[0], x.shape[1],
        _dev(first_dims, torch.int64, "first_dims"), _dev(tensor_offsets, torch.int64, "tensor_offsets"),
        _groups(first_dims, num_groups), ctypes.byref(o), _dev(status, torch.int32, "status"), _stream(stream))
    _check(rc, "nvfp4_mx_group_cast_graphsafe")


def nvfp4_mx_dequantize(data: torch.Tensor, scale: torch.Tensor, rows: int, cols: int, out: torch.Tensor,
                        stream=None) -> None:
    rc = lib().nvfp4_mx_dequantize(_dev(data, torch.uint8, "data"), _dev(scale, torch.uint8, "scale"),
                                   int(rows), int(cols), _dev(out, torch.float32, "out"), _stream(stream))
    _check(rc, "nvfp4_mx_dequantize")


def alloc_mx_outputs(rows: int, K: int, device="cuda", row: bool = True,
                     col: bool = True) -> Dict[str, torch.Tensor]:
    """Uninitialised output buffers of the grouped MXFP4 cast for ``rows`` rows."""
    out: Dict[str, torch.Tensor] = {}
    if row:
        out["row_data"] = torch.empty(rows, K // 2, dtype=torch.uint8, device=device)
        out["row_scale"] = torch.empty(rows, K // 32, dtype=torch.uint8, device=device)
    if col:
        out["col_data"] = torch.empty(rows * K // 2, dtype=torch.uint8, device=device)
        out["col_scale"] = torch.empty(rows * K // 32, dtype=torch.uint8, device=device)
    return out


def nvfp4_dequantize(data: torch.Tensor, scale: torch.Tensor, s2: torch.Tensor, rows: int, cols: int,
                     out: torch.Tensor, stream=None) -> None:
    rc = lib().nvfp4_dequantize(_dev(data, torch.uint8, "data"), _dev(scale, torch.uint8, "scale"),
                                _dev(s2, torch.float32, "s2"), int(rows), int(cols),
                                _dev(out, torch.float32, "out"), _stream(stream))
    _check(rc, "nvfp4_dequantize")


# -------------------------------------------------------- buffer helpers

def alloc_amax(rows: int, K: int, E: int, device="cuda"):
    """Uninitialised row_amax [rows] and col_amax [E*K] (fp32)."""
    return (torch.empty(rows, dtype=torch.float32, device=device),
            torch.empty(E * K, dtype=torch.float32, device=device))


def alloc_outputs(rows: int, K: int, E: int, device="cuda", row: bool = True,
                  col: bool = True) -> Dict[str, torch.Tensor]:
    """Uninitialised output buffers of the grouped cast for ``rows`` rows."""
    out: Dict[str, torch.Tensor] = {}
    if row:
        out["row_data"] = torch.empty(rows, K // 2, dtype=torch.uint8, device=device)
        out["row_scale"] = torch.empty(rows, K // 16, dtype=torch.uint8, device=device)
        out["row_s2"] = torch.empty(rows, dtype=torch.float32, device=device)
    if col:
        out["col_data"] = torch.empty(rows * K // 2, dtype=torch.uint8, device=device)
        out["col_scale"] = torch.empty(rows * K // 16, dtype=torch.uint8, device=device)
        out["col_s2"] = torch.empty(E * K, dtype=torch.float32, device=device)
    return out


def alloc_workspace(capacity_rows: int, num_groups: int, device="cuda") -> torch.Tensor:
    """Workspace of the one-launch calls (uint8; its contents need no
    initialisation, the calls zero what they use)."""
    return torch.empty(nvfp4_group_quantize_workspace_bytes(capacity_rows, num_groups),
                       dtype=torch.uint8, device=device)


def routing_tensors(m_splits: Sequence[int], K: int, device="cuda"):
    """Device first_dims [E] and tensor_offsets [E+1] (element offsets) of a
    host split list -- the graph-safe routing format."""
    fd = torch.tensor([int(m) for m in m_splits], dtype=torch.int64)
    offs = torch.zeros(len(m_splits) + 1, dtype=torch.int64)
    offs[1:] = torch.cumsum(fd, 0) * K
    return fd.to(device), offs.to(device)
