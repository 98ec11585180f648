"""Shared helpers of the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same bytes, compare byte for byte."""
import numpy as np
import torch

import oracle
from nvfp4_row_scaled_b200 import abi, workloads

KEYS = ("row_data", "row_scale", "row_s2", "col_data", "col_scale", "col_s2")


def gpu_cast(x: torch.Tensor, m_splits, rows=True, cols=True, device="cuda"):
    """Host-split amax + cast on the GPU; returns numpy copies of all outputs."""
    xd = x.to(device)
    R, K = xd.shape
    E = len(m_splits)
    ra, ca = abi.alloc_amax(R, K, E, device)
    abi.nvfp4_group_amax(xd, m_splits, ra if rows else None, ca if cols else None)
    out = abi.alloc_outputs(R, K, E, device, row=rows, col=cols)
    abi.nvfp4_group_cast(xd, m_splits, ra if rows else None, ca if cols else None, out)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    if rows:
        res["row_amax"] = ra.cpu().numpy()
    if cols:
        res["col_amax"] = ca.cpu().numpy()
    return res


def oracle_cast(x: torch.Tensor, m_splits, rows=True, cols=True):
    b = workloads.bits(x)
    ra, ca = oracle.group_amax(b, m_splits, rows=rows, cols=cols)
    out = oracle.group_cast(b, m_splits, ra, ca, rows=rows, cols=cols)
    if rows:
        out["row_amax"] = ra
    if cols:
        out["col_amax"] = ca
    return out


def same_bytes(a: np.ndarray, b: np.ndarray) -> bool:
    a = np.ascontiguousarray(a).reshape(-1)
    b = np.ascontiguousarray(b).reshape(-1)
    return a.dtype == b.dtype and a.shape == b.shape and a.view(np.uint8).tobytes() == b.view(np.uint8).tobytes()


def assert_identical(got: dict, want: dict, keys=None, what=""):
    keys = keys or [k for k in want if k in got]
    for k in keys:
        g = np.ascontiguousarray(got[k]).reshape(-1)
        w = np.ascontiguousarray(want[k]).reshape(-1)
        assert g.shape == w.shape, (what, k, g.shape, w.shape)
        gb, wb = g.view(np.uint8), w.view(np.uint8)
        if not np.array_equal(gb, wb):
            if g.dtype == np.float32:
                bad = np.nonzero(g.view(np.uint32) != w.view(np.uint32))[0]
                raise AssertionError(f"{what} {k}: {bad.size} of {g.size} differ; first at {bad[:5]}: "
                                     f"got {g[bad[:5]]} want {w[bad[:5]]}")
            bad = np.nonzero(gb != wb)[0]
            raise AssertionError(f"{what} {k}: {bad.size} of {gb.size} bytes differ; first at {bad[:5]}: "
                                 f"got {[hex(v) for v in gb[bad[:5]]]} want {[hex(v) for v in wb[bad[:5]]]}")


def special_values_case(K=256, seed=5):
    """bf16 rows with signed zeros, subnormals, exact E2M1 ties after scaling,
    tiny blocks whose scale rounds to zero, and huge and tiny magnitudes."""
    g = torch.Generator().manual_seed(seed)
    rows = []
    # row amax 6 -> enc = 1 for blocks holding a 6: x encodes as itself (ties)
    ties = torch.tensor([6, -3, 1.5, 0.25, 0.75, -0.125, 0, -0.0, 2.5, 5, 1.25, 1.75, 3.5, -6, 0.5, 4])
    r = torch.zeros(K)
    r[:16] = ties
    r[16:32] = torch.tensor([6.0] + [0.25 * k for k in range(-7, 8)])
    r[32:48] = torch.tensor([1e-7, -1e-7, 3e-8, -0.0] + [0.0] * 12)
    rows.append(r)
    # subnormal bf16 magnitudes only
    sub = (torch.randint(1, 0x80, (K,), generator=g) | (torch.randint(0, 2, (K,), generator=g) << 15))
    rows.append(sub.to(torch.int16).view(torch.bfloat16).float())
    # all zeros, all negative zeros
    rows.append(torch.zeros(K))
    rows.append(-torch.zeros(K))
    # huge range within a row
    e = torch.randint(-120, 120, (K,), generator=g).float()
    rows.append(torch.randn(K, generator=g) * torch.exp2(e))
    # near the bf16 maximum
    rows.append(torch.randn(K, generator=g).clamp(-1, 1) * 3.0e38)
    while len(rows) < 128:
        rows.append(torch.randn(K, generator=g) * float(2.0 ** int(torch.randint(-30, 30, (1,), generator=g))))
    x = torch.stack(rows).to(torch.bfloat16)
    # second group: columns of wildly different scale (colwise blocks far below the column amax)
    y = torch.randn(128, K, generator=g) * torch.exp2(torch.randint(-40, 40, (128, 1), generator=g).float())
    return torch.cat([x, y.to(torch.bfloat16)]), [128, 0, 128]


def gpu_quantize(x: torch.Tensor, m_splits, rows=True, cols=True, device="cuda", fill=None):
    """Host-split one-launch amax + cast on the GPU; numpy copies of all outputs.
    ``fill`` pre-fills every output buffer with that byte (to show that every
    byte is written)."""
    xd = x.to(device)
    R, K = xd.shape
    E = len(m_splits)
    ra, ca = abi.alloc_amax(R, K, E, device)
    out = abi.alloc_outputs(R, K, E, device, row=rows, col=cols)
    ws = abi.alloc_workspace(0, E, device)
    if fill is not None:
        for t in [ra, ca, ws, *out.values()]:
            t.view(torch.uint8).fill_(fill)
    abi.nvfp4_group_quantize(xd, m_splits, ra if rows else None, ca if cols else None, out, ws)
    torch.cuda.synchronize()
    assert int(ws[4:8].view(torch.int32).item()) == 0, "abort word raised"
    res = {k: v.cpu().numpy() for k, v in out.items()}
    if rows:
        res["row_amax"] = ra.cpu().numpy()
    if cols:
        res["col_amax"] = ca.cpu().numpy()
    return res


def host_threads() -> int:
    """Cores this process may use (the oracle releases the GIL in its calls)."""
    import os
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _eq_slice(got, want, what):
    g = np.ascontiguousarray(got).reshape(-1).view(np.uint8)
    w = np.ascontiguousarray(want).reshape(-1).view(np.uint8)
    if g.shape != w.shape or not np.array_equal(g, w):
        bad = np.nonzero(g != w)[0] if g.shape == w.shape else []
        raise AssertionError(f"{what}: {len(bad)} bytes differ, first at {list(bad[:5])}")


def check_groups_against_oracle(got: dict, xb: np.ndarray, m_splits, K: int, what: str = ""):
    """Every byte of every group's outputs (row and column amax, rowwise and
    colwise codes, scales and decode scales) against the oracle. A group's
    outputs depend on its own rows only, so the oracle runs group by group,
    spread over the host's cores; empty groups must have zero column amax and
    decode scales. ``got`` holds the GPU's buffers cut at the routed rows."""
    import concurrent.futures as cf
    offs = workloads.row_offsets(m_splits)

    def one(g):
        m, o = m_splits[g], offs[g]
        cs = slice(g * K, (g + 1) * K)
        if m == 0:
            assert np.all(got["col_amax"][cs] == 0) and np.all(got["col_s2"][cs] == 0), f"{what} empty g={g}"
            return 0
        sub = xb[o:o + m]
        ra, ca = oracle.group_amax(sub, [m])
        want = oracle.group_cast(sub, [m], ra, ca)
        tag = f"{what} g={g}"
        _eq_slice(got["row_amax"][o:o + m], ra, f"{tag} row_amax")
        _eq_slice(got["col_amax"][cs], ca, f"{tag} col_amax")
        for k in ("row_data", "row_scale", "row_s2"):
            _eq_slice(got[k][o:o + m], want[k], f"{tag} {k}")
        _eq_slice(got["col_data"][K * o // 2:K * (o + m) // 2], want["col_data"], f"{tag} col_data")
        _eq_slice(got["col_scale"][K * o // 16:K * (o + m) // 16], want["col_scale"], f"{tag} col_scale")
        _eq_slice(got["col_s2"][cs], want["col_s2"], f"{tag} col_s2")
        return m

    order = sorted(range(len(m_splits)), key=lambda g: -m_splits[g])  # largest first
    with cf.ThreadPoolExecutor(max_workers=host_threads()) as ex:
        done = sum(ex.map(one, order))
    assert done == sum(m_splits)
