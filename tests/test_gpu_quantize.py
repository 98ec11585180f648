"""The one-launch grouped amax + cast (nvfp4_group_quantize and its
graph-safe twin) on the GPU.

It must compute exactly what the two launches compute (TransformerEngine
#3649, grouped row-scaled NVFP4 cast, Description: the cast step consumes the
amax step's row and column amax vectors): every output, both amax vectors
included, byte-identical to nvfp4_group_amax + nvfp4_group_cast and to the
oracle. Cases cover many small groups (cast items that wait for their group's
amax items), empty groups, one group of many row tiles, special values, one
direction at a time, the two full-size workloads, and the graph-safe twin:
untouched tail, CUDA-graph replays with new routings, bad routing.
"""
import numpy as np
import pytest
import torch

from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import KEYS, assert_identical, gpu_cast, gpu_quantize, oracle_cast, special_values_case

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


def test_config1_against_oracle_and_two_launches():
    w = workloads.config1()
    got = gpu_quantize(w.x, w.m_splits, fill=SENTINEL)
    assert_identical(got, oracle_cast(w.x, w.m_splits), keys=ALL, what="vs oracle")
    assert_identical(got, gpu_cast(w.x, w.m_splits), keys=ALL, what="vs two launches")


@pytest.mark.parametrize("K,splits,dist,seed", [
    (128, [128], "normal", 31),
    (384, [0, 256, 128, 0], "wide", 32),
    (896, [128, 128, 128, 128, 0], "normal", 33),
    (1152, [0, 0, 1280], "heavy", 34),          # one group of ten row tiles
    (2048, [128] * 7 + [0] * 3 + [384], "normal", 35),
    (7168, [256, 0, 128, 128], "wide", 36),     # one row tile holds 56 tiles
    (256, [128] * 40, "wide", 37),              # many tiny groups
])
def test_random_cases(K, splits, dist, seed):
    w = workloads.random_case(seed, K, splits, dist=dist)
    got = gpu_quantize(w.x, splits, fill=SENTINEL)
    assert_identical(got, oracle_cast(w.x, splits), keys=ALL, what=f"K={K} {splits[:6]} vs oracle")
    assert_identical(got, gpu_cast(w.x, splits), keys=ALL, what="vs two launches")


def test_special_values():
    x, splits = special_values_case()
    assert_identical(gpu_quantize(x, splits), oracle_cast(x, splits), keys=ALL, what="special values")


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_single_direction(rows, cols):
    w = workloads.random_case(38, 640, [128, 0, 256], dist="wide")
    got = gpu_quantize(w.x, w.m_splits, rows=rows, cols=cols)
    want = oracle_cast(w.x, w.m_splits, rows=rows, cols=cols)
    assert set(got) == set(want)
    assert_identical(got, want, what=f"rows={rows} cols={cols}")


def test_repeated_calls_reuse_the_workspace():
    w = workloads.random_case(39, 1024, [256, 0, 512, 128], dist="normal")
    xd = w.x.cuda()
    R, K = xd.shape
    E = len(w.m_splits)
    ws = abi.alloc_workspace(0, E)
    ra, ca = abi.alloc_amax(R, K, E)
    out = abi.alloc_outputs(R, K, E)
    want = oracle_cast(w.x, w.m_splits)
    for _ in range(3):
        abi.nvfp4_group_quantize(xd, w.m_splits, ra, ca, out, ws)
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["row_amax"], got["col_amax"] = ra.cpu().numpy(), ca.cpu().numpy()
    assert_identical(got, want, keys=ALL, what="third call")


def test_empty_problem_and_small_workspace():
    K, E = 256, 3
    x = torch.zeros(0, K, dtype=torch.bfloat16, device="cuda")
    ra, ca = abi.alloc_amax(0, K, E)
    out = abi.alloc_outputs(0, K, E)
    out["col_s2"].fill_(7.0)
    abi.nvfp4_group_quantize(x, [0, 0, 0], ra, ca, out, abi.alloc_workspace(0, E))
    torch.cuda.synchronize()
    assert torch.all(out["col_s2"] == 0) and torch.all(ca == 0)
    small = torch.empty(abi.nvfp4_group_quantize_workspace_bytes(0, E) - 4, dtype=torch.uint8,
                        device="cuda")
    with pytest.raises(abi.NVFP4Error) as e:
        abi.nvfp4_group_quantize(x, [0, 0, 0], ra, ca, out, small)
    assert e.value.status == abi.NVFP4_ERR_INVALID_ARG


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [3, 5])
def test_full_size_matches_two_launches(cfg):
    """DeepSeek-V3-shaped MoE input and the dense 65536 x 8192 case, in the
    launch configuration the benchmark times: every byte equal to the
    two-launch path (itself checked against the oracle on samples in
    test_gpu_fullsize)."""
    w = workloads.make(cfg)
    got = gpu_quantize(w.x, w.m_splits)
    want = gpu_cast(w.x, w.m_splits)
    assert_identical(got, want, keys=ALL, what=f"config {cfg}")


# ------------------------------------------------------------ graph-safe twin

class GraphSafeQ:
    def __init__(self, x: torch.Tensor, E: int):
        self.x = x.cuda()
        self.cap, self.K = x.shape
        self.E = E
        self.fd = torch.zeros(E, dtype=torch.int64, device="cuda")
        self.offs = torch.zeros(E + 1, dtype=torch.int64, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.ws = abi.alloc_workspace(self.cap, E)
        self.ra, self.ca = abi.alloc_amax(self.cap, self.K, E)
        self.out = abi.alloc_outputs(self.cap, self.K, E)

    def set_routing(self, m_splits):
        fd, offs = abi.routing_tensors(m_splits, self.K)
        self.fd.copy_(fd)
        self.offs.copy_(offs)

    def fill(self, byte=SENTINEL):
        for t in [self.ra, self.ca, *self.out.values()]:
            t.view(torch.uint8).fill_(byte)

    def run(self):
        abi.nvfp4_group_quantize_graphsafe(self.x, self.fd, self.offs, self.ra, self.ca, self.out,
                                           self.ws, self.status)

    def results(self, total):
        K = self.K
        r = {k: v.cpu().numpy() for k, v in self.out.items()}
        r["row_amax"] = self.ra.cpu().numpy()
        r["col_amax"] = self.ca.cpu().numpy()
        cut = {"row_data": total, "row_scale": total, "row_s2": total, "row_amax": total,
               "col_data": total * K // 2, "col_scale": total * K // 16}
        return {k: (v[:cut[k]] if k in cut else v) for k, v in r.items()}, r


def test_graphsafe_byte_identical_and_untouched_tail():
    K, E, cap = 1152, 6, 1280
    splits = [256, 0, 128, 384, 0, 128]
    w = workloads.random_case(41, K, splits, capacity=cap, dist="wide")
    gs = GraphSafeQ(w.x, E)
    gs.set_routing(splits)
    gs.fill()
    gs.run()
    torch.cuda.synchronize()
    assert int(gs.status.item()) == 0
    total = sum(splits)
    got, full = gs.results(total)
    assert_identical(got, gpu_cast(w.x[:total], splits), keys=ALL, what="vs two launches")
    assert_identical(got, oracle_cast(w.x[:total], splits), keys=ALL, what="vs oracle")
    for k, cut in (("row_data", total), ("row_scale", total), ("row_s2", total), ("row_amax", total),
                   ("col_data", total * K // 2), ("col_scale", total * K // 16)):
        assert np.all(full[k][cut:].view(np.uint8) == SENTINEL), k


def test_graphsafe_cuda_graph_replays_with_ten_routings():
    w = workloads.config4(capacity=8192)
    gs = GraphSafeQ(w.x, w.E)
    gs.set_routing(w.routings[0])
    gs.run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gs.run()
    for i, splits in enumerate(w.routings):
        gs.set_routing(splits)
        gs.fill()
        graph.replay()
        torch.cuda.synchronize()
        assert int(gs.status.item()) == 0
        got, _ = gs.results(sum(splits))
        assert_identical(got, gpu_cast(w.x, splits), keys=ALL, what=f"replay {i} vs two launches")
        assert_identical(got, oracle_cast(w.x, splits), keys=ALL, what=f"replay {i} vs oracle")


@pytest.mark.parametrize("case", ["mismatch", "unaligned"])
def test_graphsafe_bad_routing_sets_status_and_writes_nothing(case):
    K, E, cap = 256, 3, 512
    w = workloads.random_case(42, K, [128, 128, 256], capacity=cap)
    gs = GraphSafeQ(w.x, E)
    fd = torch.tensor([128, 128, 256], dtype=torch.int64)
    offs = torch.tensor([0, 128, 256, 512], dtype=torch.int64) * K
    want = abi.NVFP4_ERR_ROUTING
    if case == "mismatch":
        fd[1] = 256
    else:
        fd[0], fd[1] = 64, 192
        offs[1] = 64 * K
        want = abi.NVFP4_ERR_UNSUPPORTED
    gs.fd.copy_(fd)
    gs.offs.copy_(offs)
    gs.fill()
    gs.run()
    torch.cuda.synchronize()
    assert int(gs.status.item()) == want
    full = gs.results(0)[1]
    for k in ("row_data", "row_scale", "row_s2", "row_amax", "col_data", "col_scale", "col_s2"):
        assert np.all(full[k].view(np.uint8) == SENTINEL), k
    gs.set_routing([128, 128, 256])
    gs.run()
    torch.cuda.synchronize()
    assert int(gs.status.item()) == 0


def test_graphsafe_full_capacity_config4_replays():
    w = workloads.config4()
    gs = GraphSafeQ(w.x, w.E)
    gs.set_routing(w.routings[0])
    gs.run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gs.run()
    for i, splits in enumerate(w.routings):
        gs.set_routing(splits)
        graph.replay()
        torch.cuda.synchronize()
        assert int(gs.status.item()) == 0
        got, _ = gs.results(sum(splits))
        assert_identical(got, gpu_cast(w.x, splits), keys=ALL, what=f"full replay {i}")
