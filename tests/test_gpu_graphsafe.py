"""Graph-safe path on the GPU: routing read from device first_dims /
tensor_offsets (TransformerEngine #3649, grouped row-scaled NVFP4 cast,
Description).

- byte-identical to the host-split path for equal routing;
- rows at or beyond the routed total are neither read nor written;
- captured once in a CUDA graph and replayed with new routings written into
  the same device buffers, each replay checked against the oracle and the
  host-split call;
- inconsistent routing sets the status word and writes nothing; no trap.
"""
import numpy as np
import pytest
import torch

from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import KEYS, assert_identical, check_groups_against_oracle, gpu_cast, oracle_cast

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


class GraphSafe:
    """Buffers of one graph-safe problem: capacity rows, E groups."""

    def __init__(self, x: torch.Tensor, E: int):
        self.x = x.cuda()
        self.cap, self.K = x.shape
        self.E = E
        self.fd = torch.zeros(E, dtype=torch.int64, device="cuda")
        self.offs = torch.zeros(E + 1, dtype=torch.int64, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
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
        abi.nvfp4_group_amax_graphsafe(self.x, self.fd, self.offs, self.ra, self.ca, self.status)
        abi.nvfp4_group_cast_graphsafe(self.x, self.fd, self.offs, self.ra, self.ca, self.out,
                                       self.status)

    def results(self, total):
        """Outputs of the routed rows, as numpy (rowwise buffers cut at total)."""
        K = self.K
        r = {k: v.cpu().numpy() for k, v in self.out.items()}
        r["row_amax"] = self.ra.cpu().numpy()
        r["col_amax"] = self.ca.cpu().numpy()
        cut = {"row_data": total, "row_scale": total, "row_s2": total, "row_amax": total,
               "col_data": total * K // 2, "col_scale": total * K // 16}
        return {k: (v[:cut[k]] if k in cut else v) for k, v in r.items()}, r


def test_byte_identical_to_host_split_and_untouched_tail():
    K, E, cap = 1152, 6, 1280
    splits = [256, 0, 128, 384, 0, 128]  # 896 routed rows of 1280
    w = workloads.random_case(21, K, splits, capacity=cap, dist="wide")
    gs = GraphSafe(w.x, E)
    gs.set_routing(splits)
    gs.fill()
    gs.run()
    torch.cuda.synchronize()
    assert int(gs.status.item()) == 0
    total = sum(splits)
    got, full = gs.results(total)
    host = gpu_cast(w.x[:total], splits)
    assert_identical(got, host, what="graph-safe vs host-split")
    assert_identical(got, oracle_cast(w.x[:total], splits), what="graph-safe vs oracle")
    # nothing beyond the routed rows was written
    assert np.all(full["row_data"][total:] == SENTINEL)
    assert np.all(full["row_scale"][total:] == SENTINEL)
    assert np.all(full["row_s2"][total:].view(np.uint8) == SENTINEL)
    assert np.all(full["row_amax"][total:].view(np.uint8) == SENTINEL)
    assert np.all(full["col_data"][total * K // 2:] == SENTINEL)
    assert np.all(full["col_scale"][total * K // 16:] == SENTINEL)


def test_cuda_graph_capture_and_replay_with_ten_routings():
    """Config-4 recipe at reduced capacity so every replay is checked
    against the oracle in full."""
    w = workloads.config4(capacity=8192)
    gs = GraphSafe(w.x, w.E)
    gs.set_routing(w.routings[0])
    gs.run()  # warm up (loads the kernels) outside the capture
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
        assert_identical(got, gpu_cast(w.x, splits), what=f"replay {i} vs host-split")
        assert_identical(got, oracle_cast(w.x, splits), what=f"replay {i} vs oracle")


@pytest.mark.parametrize("case", ["offset0", "mismatch", "beyond_capacity", "negative", "unaligned"])
def test_bad_device_routing_sets_status_and_writes_nothing(case):
    K, E, cap = 256, 3, 512
    w = workloads.random_case(22, K, [128, 128, 256], capacity=cap)
    gs = GraphSafe(w.x, E)
    fd = torch.tensor([128, 128, 256], dtype=torch.int64)
    offs = torch.tensor([0, 128, 256, 512], dtype=torch.int64) * K
    want = abi.NVFP4_ERR_ROUTING
    if case == "offset0":
        offs += K * 128
    elif case == "mismatch":
        fd[1] = 256
    elif case == "beyond_capacity":
        fd[2] = 384
        offs[3] = 640 * K
    elif case == "negative":
        fd[0], fd[1] = -128, 384
        offs[1] = -128 * K
    elif case == "unaligned":  # a group that is not a multiple of 16 rows
        fd[0], fd[1] = 72, 184
        offs[1] = 72 * K
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
    # col_amax was zeroed by the amax call before its kernel saw the routing
    assert np.all(full["col_amax"] == 0)
    # the context is still usable: a good routing afterwards works
    gs.set_routing([128, 128, 256])
    gs.run()
    torch.cuda.synchronize()
    assert int(gs.status.item()) == 0


def test_config4_full_capacity_replays_match_host_split_and_oracle():
    """Full-size config 4 (131072 x 2048, 128 experts): every one of the ten
    graph replays is byte-identical to the host-split call and, in full, to
    the oracle (run group by group over the host's cores)."""
    w = workloads.config4()
    gs = GraphSafe(w.x, w.E)
    gs.set_routing(w.routings[0])
    gs.run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gs.run()
    xb = workloads.bits(w.x)
    for i, splits in enumerate(w.routings):
        gs.set_routing(splits)
        graph.replay()
        torch.cuda.synchronize()
        assert int(gs.status.item()) == 0
        got, _ = gs.results(sum(splits))
        assert_identical(got, gpu_cast(w.x, splits), keys=list(KEYS) + ["row_amax", "col_amax"],
                         what=f"full replay {i}")
        check_groups_against_oracle(got, xb, splits, w.K, what=f"full replay {i}")
