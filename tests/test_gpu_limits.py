"""Limits on the GPU: the largest group count (NVFP4_MAX_GROUPS = 1024, most
of them empty, where the kernels' shared routing tables are largest), a
single group, and a wide K, through every cast path, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import KEYS, assert_identical, gpu_cast, gpu_quantize, oracle_cast

pytestmark = pytest.mark.gpu

ALL = list(KEYS) + ["row_amax", "col_amax"]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


def max_groups_splits():
    E = abi.NVFP4_MAX_GROUPS
    splits = [0] * E
    for g, m in ((0, 128), (3, 256), (511, 128), (1000, 128), (E - 1, 128)):
        splits[g] = m
    return splits


def test_max_groups_every_path():
    splits = max_groups_splits()
    K = 256
    w = workloads.random_case(120, K, splits, dist="wide")
    want = oracle_cast(w.x, splits)
    assert_identical(gpu_cast(w.x, splits), want, keys=ALL, what="two launches")
    assert_identical(gpu_quantize(w.x, splits), want, keys=ALL, what="one launch")
    # graph-safe two-step
    x = w.x.cuda()
    R = x.shape[0]
    fd, offs = abi.routing_tensors(splits, K)
    ra, ca = abi.alloc_amax(R, K, len(splits))
    out = abi.alloc_outputs(R, K, len(splits))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.nvfp4_group_amax_graphsafe(x, fd, offs, ra, ca, st)
    abi.nvfp4_group_cast_graphsafe(x, fd, offs, ra, ca, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["row_amax"], got["col_amax"] = ra.cpu().numpy(), ca.cpu().numpy()
    assert_identical(got, want, keys=ALL, what="graph-safe")
    # MXFP4
    mx = abi.alloc_mx_outputs(R, K)
    abi.nvfp4_mx_group_cast(x, splits, mx)
    torch.cuda.synchronize()
    mw = oracle.mx_group_cast(workloads.bits(w.x), splits)
    for k, v in mw.items():
        assert np.array_equal(mx[k].cpu().numpy(), v), k


@pytest.mark.parametrize("K", [128, 16384])
def test_single_group_and_wide_k(K):
    splits = [256]
    w = workloads.random_case(121 + K, K, splits, dist="heavy")
    want = oracle_cast(w.x, splits)
    assert_identical(gpu_cast(w.x, splits), want, keys=ALL, what=f"K={K}")
    assert_identical(gpu_quantize(w.x, splits), want, keys=ALL, what=f"one launch K={K}")
