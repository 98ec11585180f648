"""Groups whose sizes are multiples of 16 rows but not of 128, K that is a
multiple of 16 but not of 128, and uniform groups, on the GPU (the
robustness the TransformerEngine #3649 review asks for: supported shapes
beyond the 128-row-aligned grouped fast path, and uniform expert sizes).

Group sizes only need to be multiples of 16 (the colwise block height), so a
16-row block always lies in one group; a 128-row tile may hold rows of
several groups, and the last tile may be short. K only needs to be a
multiple of 16 (the rowwise block width); the last 128-column tile may then
be partial. Checked byte for byte against the oracle, host-split and
graph-safe (which must also agree with each other, and leave every byte past
the routed rows untouched), in both directions and in each alone; uniform
graph-safe routing (no first_dims / tensor_offsets); the host-split
one-launch calls, whose single launch keeps 128-row groups and K % 128 == 0,
run the rest as the two launches.
"""
import numpy as np
import pytest
import torch

from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import KEYS, assert_identical, check_groups_against_oracle, gpu_cast, oracle_cast, \
    special_values_case

pytestmark = pytest.mark.gpu

ALL = list(KEYS) + ["row_amax", "col_amax"]
SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


CASES = [
    (128, [16], "normal", 61),                           # one short tile
    (256, [48, 0, 16, 144, 32], "wide", 62),             # several groups per tile, empty in the middle
    (384, [16] * 9 + [0, 0] + [80], "heavy", 63),        # many tiny groups
    (896, [272, 400, 0, 112], "normal", 64),             # groups straddling tiles, short tail
    (1152, [0, 0, 144], "wide", 65),                     # one group, not a multiple of 128
    (7168, [208, 0, 48, 96], "wide", 66),
    (256, [16, 256, 112], "normal", 70),                 # a 128-multiple group starting at row 16
]


@pytest.mark.parametrize("K,splits,dist,seed", CASES)
def test_unaligned_against_oracle(K, splits, dist, seed):
    w = workloads.random_case(seed, K, splits, dist=dist)
    assert_identical(gpu_cast(w.x, splits), oracle_cast(w.x, splits), keys=ALL,
                     what=f"K={K} {splits}")


KCASES = [
    (16, [128, 16], "normal", 80),       # K below one TMA box: one 16-column tile
    (48, [32, 0, 96], "wide", 81),       # second TMA box wholly past K
    (144, [256], "normal", 82),          # one full and one 16-column tile per row tile
    (528, [48, 208, 16], "wide", 83),    # K = 4*128 + 16 with unaligned groups
    (2064, [384, 128], "heavy", 84),     # 128-aligned groups, partial last column tile
    (7184, [0, 256, 112], "wide", 85),   # DeepSeek-V3 hidden size + 16
]


@pytest.mark.parametrize("K,splits,dist,seed", KCASES)
def test_k_not_multiple_of_128_against_oracle(K, splits, dist, seed):
    w = workloads.random_case(seed, K, splits, dist=dist)
    assert_identical(gpu_cast(w.x, splits), oracle_cast(w.x, splits), keys=ALL,
                     what=f"K={K} {splits}")


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_k_not_multiple_of_128_single_direction(rows, cols):
    splits = [48, 0, 208, 16]
    w = workloads.random_case(86, 400, splits, dist="wide")
    got = gpu_cast(w.x, splits, rows=rows, cols=cols)
    want = oracle_cast(w.x, splits, rows=rows, cols=cols)
    assert set(got) == set(want)
    assert_identical(got, want)


def test_k_not_multiple_of_128_special_values():
    x, _ = special_values_case(K=400)
    splits = [48, 0, 80, 16, 112]
    assert_identical(gpu_cast(x, splits), oracle_cast(x, splits), keys=ALL, what="special values K=400")


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_unaligned_single_direction(rows, cols):
    splits = [48, 0, 208, 16]
    w = workloads.random_case(67, 640, splits, dist="wide")
    got = gpu_cast(w.x, splits, rows=rows, cols=cols)
    want = oracle_cast(w.x, splits, rows=rows, cols=cols)
    assert set(got) == set(want)
    assert_identical(got, want)


def test_unaligned_special_values():
    x, _ = special_values_case()
    splits = [48, 0, 80, 16, 112]  # the same 256 rows cut at 16-row boundaries
    assert_identical(gpu_cast(x, splits), oracle_cast(x, splits), keys=ALL, what="special values")


def test_deepseek_shape_padded_to_16():
    """DeepSeek-V3-shaped routing with groups padded to 16 rows (1024
    tokens): every output byte against the oracle."""
    w = workloads.config3(tokens=1024, align=16)
    assert any(m % 128 for m in w.m_splits)
    assert_identical(gpu_cast(w.x, w.m_splits), oracle_cast(w.x, w.m_splits), keys=ALL, what=w.name)


def graphsafe(x, E, fd=None, offs=None, num_groups=None, fill=True):
    cap, K = x.shape
    ra, ca = abi.alloc_amax(cap, K, E)
    out = abi.alloc_outputs(cap, K, E)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if fill:
        for t in [ra, ca, *out.values()]:
            t.view(torch.uint8).fill_(SENTINEL)
    abi.nvfp4_group_amax_graphsafe(x, fd, offs, ra, ca, status, num_groups=num_groups)
    abi.nvfp4_group_cast_graphsafe(x, fd, offs, ra, ca, out, status, num_groups=num_groups)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["row_amax"], res["col_amax"] = ra.cpu().numpy(), ca.cpu().numpy()
    return res, int(status.item())


def cut(res, total, K):
    c = {"row_data": total, "row_scale": total, "row_s2": total, "row_amax": total,
         "col_data": total * K // 2, "col_scale": total * K // 16}
    return {k: (v[:c[k]] if k in c else v) for k, v in res.items()}


def test_graphsafe_unaligned_matches_host_split_and_leaves_tail():
    K, cap = 384, 640
    splits = [48, 0, 208, 16, 112]  # 384 routed rows of 640
    w = workloads.random_case(68, K, splits, capacity=cap, dist="wide")
    x = w.x.cuda()
    fd, offs = abi.routing_tensors(splits, K)
    full, st = graphsafe(x, len(splits), fd, offs)
    assert st == 0
    total = sum(splits)
    got = cut(full, total, K)
    assert_identical(got, gpu_cast(w.x[:total], splits), keys=ALL, what="vs host-split")
    assert_identical(got, oracle_cast(w.x[:total], splits), keys=ALL, what="vs oracle")
    for k, c in (("row_data", total), ("row_scale", total), ("row_s2", total), ("row_amax", total),
                 ("col_data", total * K // 2), ("col_scale", total * K // 16)):
        assert np.all(full[k][c:].view(np.uint8) == SENTINEL), k


def test_graphsafe_k_not_multiple_of_128_matches_host_split_and_leaves_tail():
    K, cap = 656, 512
    splits = [16, 0, 208, 112]  # 336 routed rows of 512
    w = workloads.random_case(87, K, splits, capacity=cap, dist="wide")
    x = w.x.cuda()
    fd, offs = abi.routing_tensors(splits, K)
    full, st = graphsafe(x, len(splits), fd, offs)
    assert st == 0
    total = sum(splits)
    got = cut(full, total, K)
    assert_identical(got, gpu_cast(w.x[:total], splits), keys=ALL, what="vs host-split")
    assert_identical(got, oracle_cast(w.x[:total], splits), keys=ALL, what="vs oracle")
    for k, c in (("row_data", total), ("row_scale", total), ("row_s2", total), ("row_amax", total),
                 ("col_data", total * K // 2), ("col_scale", total * K // 16)):
        assert np.all(full[k][c:].view(np.uint8) == SENTINEL), k


def test_tiled_layout_refuses_k_not_multiple_of_128():
    K = 144
    splits = [128, 128]
    x = torch.zeros(256, K, dtype=torch.bfloat16, device="cuda")
    ra, ca = abi.alloc_amax(256, K, 2)
    out = abi.alloc_outputs(256, K, 2)
    for call in (lambda: abi.nvfp4_group_cast(x, splits, ra, ca, out, scale_layout=abi.NVFP4_SCALE_TILED_128X4),
                 lambda: abi.nvfp4_group_quantize(x, splits, ra, ca, out, abi.alloc_workspace(0, 2),
                                                  scale_layout=abi.NVFP4_SCALE_TILED_128X4)):
        with pytest.raises(abi.NVFP4Error) as e:
            call()
        assert e.value.status == abi.NVFP4_ERR_UNSUPPORTED


ONE_LAUNCH_CASES = [CASES[1], CASES[3], CASES[6], KCASES[0], KCASES[3], KCASES[4]]


@pytest.mark.parametrize("K,splits,dist,seed", ONE_LAUNCH_CASES)
def test_one_launch_calls_take_every_routing(K, splits, dist, seed):
    """The host-split one-launch calls run a routing their single launch does
    not take (groups off the 128-row grid, K % 128 != 0) as the two launches:
    byte-identical to the oracle, workspace untouched."""
    w = workloads.random_case(seed, K, splits, dist=dist)
    want = oracle_cast(w.x, splits)
    xd = w.x.cuda()
    R, E = xd.shape[0], len(splits)
    for name in ("workspace", "noalloc"):
        ra, ca = abi.alloc_amax(R, K, E)
        out = abi.alloc_outputs(R, K, E)
        for t in [ra, ca, *out.values()]:
            t.view(torch.uint8).fill_(SENTINEL)
        if name == "workspace":
            ws = abi.alloc_workspace(0, E)
            ws.fill_(SENTINEL)
            abi.nvfp4_group_quantize(xd, splits, ra, ca, out, ws)
        else:
            abi.nvfp4_group_quantize_noalloc(xd, splits, ra, ca, out)
        torch.cuda.synchronize()
        got = {k: v.cpu().numpy() for k, v in out.items()}
        got["row_amax"], got["col_amax"] = ra.cpu().numpy(), ca.cpu().numpy()
        assert_identical(got, want, keys=ALL, what=f"{name} K={K} {splits}")
        if name == "workspace":
            assert bool((ws == SENTINEL).all()), "the two-launch path leaves the workspace untouched"


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_one_launch_calls_unaligned_single_direction(rows, cols):
    splits = [48, 0, 208, 16]
    w = workloads.random_case(87, 400, splits, dist="wide")
    xd = w.x.cuda()
    R, K, E = xd.shape[0], xd.shape[1], len(splits)
    ra, ca = abi.alloc_amax(R, K, E)
    out = abi.alloc_outputs(R, K, E, row=rows, col=cols)
    abi.nvfp4_group_quantize(xd, splits, ra if rows else None, ca if cols else None, out,
                             abi.alloc_workspace(0, E))
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in out.items()}
    if rows:
        got["row_amax"] = ra.cpu().numpy()
    if cols:
        got["col_amax"] = ca.cpu().numpy()
    want = oracle_cast(w.x, splits, rows=rows, cols=cols)
    assert_identical(got, want, keys=list(want.keys()), what=f"rows={rows} cols={cols}")


@pytest.mark.parametrize("E,m", [(4, 128), (10, 48)])
def test_graphsafe_uniform_groups(E, m):
    K = 256
    splits = [m] * E
    w = workloads.random_case(69 + E, K, splits, dist="normal")
    x = w.x.cuda()
    res, st = graphsafe(x, E, num_groups=E)
    assert st == 0
    assert_identical(res, gpu_cast(w.x, splits), keys=ALL, what="uniform vs host-split")
    assert_identical(res, oracle_cast(w.x, splits), keys=ALL, what="uniform vs oracle")


def test_uniform_groups_must_divide_capacity():
    x = torch.zeros(100, 128, dtype=torch.bfloat16, device="cuda")
    ra, ca = abi.alloc_amax(100, 128, 3)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(abi.NVFP4Error) as e:
        abi.nvfp4_group_amax_graphsafe(x, None, None, ra, ca, status, num_groups=3)
    assert e.value.status == abi.NVFP4_ERR_INVALID_ARG


def test_graphsafe_group_not_multiple_of_16_is_unsupported():
    K, cap = 128, 256
    x = torch.zeros(cap, K, dtype=torch.bfloat16, device="cuda")
    fd = torch.tensor([40, 88], dtype=torch.int64, device="cuda")
    offs = torch.tensor([0, 40 * K, 128 * K], dtype=torch.int64, device="cuda")
    full, st = graphsafe(x, 2, fd, offs)
    assert st == abi.NVFP4_ERR_UNSUPPORTED
    for k in KEYS:
        assert np.all(full[k].view(np.uint8) == SENTINEL), k


def test_graphsafe_one_launch_refuses_unaligned_groups():
    """The graph-safe one-launch call keeps its single launch and 128-row
    groups: the device routing check reports the rest."""
    K = 256
    splits = [48, 208]
    x = torch.zeros(sum(splits), K, dtype=torch.bfloat16, device="cuda")
    ra, ca = abi.alloc_amax(sum(splits), K, 2)
    out = abi.alloc_outputs(sum(splits), K, 2)
    fd, offs = abi.routing_tensors(splits, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.nvfp4_group_quantize_graphsafe(x, fd, offs, ra, ca, out, abi.alloc_workspace(sum(splits), 2), status)
    torch.cuda.synchronize()
    assert int(status.item()) == abi.NVFP4_ERR_UNSUPPORTED


@pytest.mark.slow
def test_deepseek_shape_padded_to_16_full_size():
    """Full DeepSeek-V3 routing (8192 tokens) padded to 16 rows, in the
    benchmark's launch configuration: every byte of every group against the
    oracle (run group by group over the host's cores)."""
    w = workloads.config3(align=16)
    assert any(m % 128 for m in w.m_splits)
    check_groups_against_oracle(gpu_cast(w.x, w.m_splits), workloads.bits(w.x), w.m_splits, w.K,
                                what="deepseek-v3 padded to 16")
