"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar: bit-exact on every output -- amax values, FP4 bytes, E4M3 scale bytes
and FP32 decode scales (compared as bit patterns), both directions. Cases
span several tiles, every cluster width of the amax kernel (K/128 = 1, 3, 5,
7, 8, 9, 16, 56), a partial column group in the cast (K/128 not a multiple of
4), empty groups at the front, middle and end, and special values (signed
zeros, subnormals, exact E2M1 ties, blocks whose scale rounds to zero, values
near the bf16 maximum).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import assert_identical, gpu_cast, oracle_cast, special_values_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


def test_config1_tiny_grouped_cast():
    w = workloads.config1()
    assert_identical(gpu_cast(w.x, w.m_splits), oracle_cast(w.x, w.m_splits), what=w.name)


@pytest.mark.parametrize("K,splits,dist,seed", [
    (128, [128], "normal", 1),
    (384, [0, 256, 128, 0], "wide", 2),
    (640, [384, 0, 128], "heavy", 3),
    (896, [128, 128, 128, 128, 0], "normal", 4),
    (1024, [256, 512], "wide", 5),
    (1152, [0, 0, 640], "heavy", 6),
    (2048, [128] * 7 + [0] * 3 + [384], "normal", 7),
    (7168, [256, 0, 128], "wide", 8),
])
def test_random_cases(K, splits, dist, seed):
    w = workloads.random_case(seed, K, splits, dist=dist)
    assert_identical(gpu_cast(w.x, splits), oracle_cast(w.x, splits), what=f"K={K} {splits} {dist}")


def test_special_values():
    x, splits = special_values_case()
    assert_identical(gpu_cast(x, splits), oracle_cast(x, splits), what="special values")


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_single_direction(rows, cols):
    w = workloads.random_case(9, 640, [128, 0, 256], dist="wide")
    got = gpu_cast(w.x, w.m_splits, rows=rows, cols=cols)
    want = oracle_cast(w.x, w.m_splits, rows=rows, cols=cols)
    assert_identical(got, want, what=f"rows={rows} cols={cols}")


def test_many_groups_and_empty_problem():
    E = 1024
    splits = [0] * E
    splits[3], splits[500], splits[1023] = 128, 256, 128
    w = workloads.random_case(10, 128, splits)
    assert_identical(gpu_cast(w.x, splits), oracle_cast(w.x, splits), what="E=1024")
    # no rows at all: col amax / col_s2 are zeros, nothing else is written
    x0 = torch.zeros(0, 256, dtype=torch.bfloat16)
    got = gpu_cast(x0, [0, 0, 0])
    assert np.all(got["col_amax"] == 0) and np.all(got["col_s2"] == 0)


def test_config2_outlier_rows_full():
    w = workloads.config2()
    assert_identical(gpu_cast(w.x, w.m_splits), oracle_cast(w.x, w.m_splits), what=w.name)


def test_dequantize_matches_oracle_both_directions():
    w = workloads.random_case(11, 640, [256, 0, 128], dist="heavy")
    K = w.K
    xd = w.x.cuda()
    R = xd.shape[0]
    ra, ca = abi.alloc_amax(R, K, w.E)
    abi.nvfp4_group_amax(xd, w.m_splits, ra, ca)
    out = abi.alloc_outputs(R, K, w.E)
    abi.nvfp4_group_cast(xd, w.m_splits, ra, ca, out)
    xh = torch.empty(R, K, dtype=torch.float32, device="cuda")
    abi.nvfp4_dequantize(out["row_data"], out["row_scale"], out["row_s2"], R, K, xh)
    o = {k: v.cpu().numpy() for k, v in out.items()}
    want = oracle.dequantize(o["row_data"], o["row_scale"], o["row_s2"], R, K)
    assert_identical({"x": xh.cpu().numpy()}, {"x": want}, what="rowwise dequant")
    offs = workloads.row_offsets(w.m_splits)
    for g, m in enumerate(w.m_splits):
        if m == 0:
            continue
        d = out["col_data"][K * offs[g] // 2: K * (offs[g] + m) // 2]
        s = out["col_scale"][K * offs[g] // 16: K * (offs[g] + m) // 16]
        s2 = out["col_s2"][g * K:(g + 1) * K]
        xh = torch.empty(K, m, dtype=torch.float32, device="cuda")
        abi.nvfp4_dequantize(d, s, s2, K, m, xh)
        want = oracle.dequantize(d.cpu().numpy(), s.cpu().numpy(), s2.cpu().numpy(), K, m)
        assert_identical({"x": xh.cpu().numpy()}, {"x": want}, what=f"colwise dequant g={g}")


@pytest.mark.parametrize("K,splits", [(7168, [256, 0, 384, 128]), (2048, [48, 208, 16, 0, 112]), (144, [128, 32])])
def test_amax_waits_for_its_zeroing(K, splits):
    """col_amax starts as all-ones words (larger, as unsigned, than any float
    the atomic max can bring): the amax call's zeroing kernel must finish
    before the first atomic of the amax kernel launched programmatically
    after it, on every call (TransformerEngine #3649, Description: the amax
    step's column amax vector is the per-group maximum)."""
    w = workloads.random_case(91, K, splits, dist="wide")
    want = oracle_cast(w.x, splits)
    xd = w.x.cuda()
    R, E = xd.shape[0], len(splits)
    ra, ca = abi.alloc_amax(R, K, E)
    for call in range(3):
        ca.view(torch.int32).fill_(-1)
        ra.view(torch.int32).fill_(-1)
        abi.nvfp4_group_amax(xd, splits, ra, ca)
        torch.cuda.synchronize()
        assert_identical({"row_amax": ra.cpu().numpy(), "col_amax": ca.cpu().numpy()}, want,
                         keys=["row_amax", "col_amax"], what=f"call {call}")
    fd, offs = abi.routing_tensors(splits, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ca.view(torch.int32).fill_(-1)
    abi.nvfp4_group_amax_graphsafe(xd, fd, offs, ra, ca, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_identical({"col_amax": ca.cpu().numpy()}, want, keys=["col_amax"], what="graph-safe")
