"""nvfp4_group_quantize_noalloc on the GPU: the one-launch kernel with its
scratch in the library's static device array, called through the C ABI.

Checked against the entry point that takes a workspace
(nvfp4_group_quantize): every output and both amax vectors must match
exactly (the encodings are integer codes and exactly rounded scales, so the
tolerance is zero), on two calls in a row -- the second call reuses the
static scratch the first one left behind. This file is collected last so it
also runs after every other GPU test in the same process.
"""
import pytest
import torch

from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import KEYS, assert_identical

pytestmark = pytest.mark.gpu

ALL = list(KEYS) + ["row_amax", "col_amax"]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


def run(fn, x, splits):
    R, K = x.shape
    E = len(splits)
    ra, ca = abi.alloc_amax(R, K, E)
    out = abi.alloc_outputs(R, K, E)
    for t in [ra, ca, *out.values()]:
        t.view(torch.uint8).fill_(0xA5)
    fn(ra, ca, out)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["row_amax"], res["col_amax"] = ra.cpu().numpy(), ca.cpu().numpy()
    return res


@pytest.mark.parametrize("case", ["config1", "empty_groups", "deepseek_t1024"])
def test_noalloc_matches_workspace_call_twice_in_a_row(case):
    if case == "config1":
        w = workloads.config1()
    elif case == "empty_groups":
        w = workloads.random_case(51, 1024, [0, 256, 0, 128, 384, 0], dist="wide")
    else:
        w = workloads.config3(tokens=1024)
    x = w.x.cuda()
    splits = w.m_splits
    ws = abi.alloc_workspace(0, len(splits))
    want = run(lambda ra, ca, out: abi.nvfp4_group_quantize(x, splits, ra, ca, out, ws), x, splits)
    for call in range(2):
        got = run(lambda ra, ca, out: abi.nvfp4_group_quantize_noalloc(x, splits, ra, ca, out), x, splits)
        assert_identical(got, want, keys=ALL, what=f"{case} call {call}")


def test_noalloc_rejects_more_groups_than_its_scratch_holds():
    K = 128
    E = abi.NVFP4_MAX_GROUPS + 1
    x = torch.zeros(128, K, dtype=torch.bfloat16, device="cuda")
    splits = [128] + [0] * (E - 1)
    ra, ca = abi.alloc_amax(128, K, E)
    out = abi.alloc_outputs(128, K, E)
    with pytest.raises(abi.NVFP4Error) as e:
        abi.nvfp4_group_quantize_noalloc(x, splits, ra, ca, out)
    assert e.value.status == abi.NVFP4_ERR_UNSUPPORTED
