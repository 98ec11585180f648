"""Grouped MXFP4 cast on the GPU (E2M1, blocks of 32, E8M0 scales; the
"E2M1/block-32/E8M0" configuration of TransformerEngine #3824, Testing),
byte for byte against the oracle: both directions and each alone, empty
groups, several widths, groups of any multiple of 32 rows and K any multiple
of 32, special values (zeros, subnormals, ties, values near the bf16
maximum), the graph-safe twin (identical, untouched tail, refused routing),
and the MXFP4 dequantize (bit-exact fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import special_values_case

pytestmark = pytest.mark.gpu

MX_KEYS = ("row_data", "row_scale", "col_data", "col_scale")


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


def gpu_mx(x, splits, rows=True, cols=True):
    xd = x.cuda()
    R, K = xd.shape
    out = abi.alloc_mx_outputs(R, K, row=rows, col=cols)
    for t in out.values():
        t.fill_(0xA5)
    abi.nvfp4_mx_group_cast(xd, splits, out)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def check(got, want, what=""):
    assert set(got) == set(want), what
    for k in want:
        g, w = np.asarray(got[k]).reshape(-1), np.asarray(want[k]).reshape(-1)
        if not np.array_equal(g, w):
            bad = np.nonzero(g != w)[0]
            raise AssertionError(f"{what} {k}: {bad.size} of {g.size} bytes differ, first at {bad[:5]}: "
                                 f"got {g[bad[:5]]} want {w[bad[:5]]}")


def test_config1():
    w = workloads.config1()
    check(gpu_mx(w.x, w.m_splits), oracle.mx_group_cast(workloads.bits(w.x), w.m_splits), "config1")


@pytest.mark.parametrize("K,splits,dist,seed", [
    (128, [128], "normal", 101),
    (384, [0, 256, 128, 0], "wide", 102),
    (1152, [384, 0, 128], "heavy", 103),
    (7168, [256, 0, 128], "wide", 104),
])
def test_random_cases(K, splits, dist, seed):
    w = workloads.random_case(seed, K, splits, dist=dist)
    check(gpu_mx(w.x, splits), oracle.mx_group_cast(workloads.bits(w.x), splits), f"K={K} {splits}")


def test_special_values():
    x, splits = special_values_case()
    check(gpu_mx(x, splits), oracle.mx_group_cast(workloads.bits(x), splits), "special values")


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_single_direction(rows, cols):
    w = workloads.random_case(105, 640, [128, 0, 256], dist="wide")
    check(gpu_mx(w.x, w.m_splits, rows, cols),
          oracle.mx_group_cast(workloads.bits(w.x), w.m_splits, rows, cols), f"rows={rows}")


def test_graphsafe_identical_and_tail_untouched():
    K, cap = 512, 768
    splits = [256, 0, 128]
    w = workloads.random_case(106, K, splits, capacity=cap, dist="wide")
    x = w.x.cuda()
    fd, offs = abi.routing_tensors(splits, K)
    out = abi.alloc_mx_outputs(cap, K)
    for t in out.values():
        t.fill_(0xA5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.nvfp4_mx_group_cast_graphsafe(x, fd, offs, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    total = sum(splits)
    got = {k: v.cpu().numpy() for k, v in out.items()}
    cut = {"row_data": total, "row_scale": total, "col_data": total * K // 2, "col_scale": total * K // 32}
    head = {k: v[:cut[k]] for k, v in got.items()}
    check(head, gpu_mx(w.x[:total], splits), "graph-safe vs host-split")
    for k, v in got.items():
        assert np.all(v[cut[k]:] == 0xA5), k


def test_graphsafe_refuses_groups_off_the_32_row_grid():
    K = 256
    x = torch.zeros(256, K, dtype=torch.bfloat16, device="cuda")
    fd = torch.tensor([48, 208], dtype=torch.int64, device="cuda")
    offs = torch.tensor([0, 48 * K, 256 * K], dtype=torch.int64, device="cuda")
    out = abi.alloc_mx_outputs(256, K)
    for t in out.values():
        t.fill_(0xA5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.nvfp4_mx_group_cast_graphsafe(x, fd, offs, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == abi.NVFP4_ERR_UNSUPPORTED
    for k, v in out.items():
        assert bool(torch.all(v == 0xA5)), k
    with pytest.raises(abi.NVFP4Error) as e:
        abi.nvfp4_mx_group_cast(x, [48, 208], out)
    assert e.value.status == abi.NVFP4_ERR_UNSUPPORTED


# groups of any multiple of 32 rows and K any multiple of 32: tiles that a
# group boundary crosses, groups off the 128-row grid, a short last row tile,
# a partial last column tile
UNALIGNED = [
    (128, [32], "normal", 111),                        # one short tile
    (256, [96, 0, 32, 160, 64], "wide", 112),          # several groups per tile, empty in the middle
    (160, [128, 32, 0, 96], "heavy", 113),             # K = 128 + 32
    (32, [64, 224], "normal", 114),                    # K below one TMA box
    (1056, [288, 0, 416, 96], "wide", 115),            # K = 8*128 + 32, groups straddling tiles
    (7168, [224, 0, 32, 96], "wide", 116),
]


@pytest.mark.parametrize("K,splits,dist,seed", UNALIGNED)
def test_unaligned_groups_and_k(K, splits, dist, seed):
    w = workloads.random_case(seed, K, splits, dist=dist)
    check(gpu_mx(w.x, splits), oracle.mx_group_cast(workloads.bits(w.x), splits), f"K={K} {splits}")


@pytest.mark.parametrize("rows,cols", [(True, False), (False, True)])
def test_unaligned_single_direction(rows, cols):
    splits = [96, 0, 224, 32]
    w = workloads.random_case(117, 416, splits, dist="wide")
    check(gpu_mx(w.x, splits, rows, cols), oracle.mx_group_cast(workloads.bits(w.x), splits, rows, cols),
          f"rows={rows}")


def test_unaligned_special_values():
    x, _ = special_values_case(K=416)
    splits = [96, 0, 64, 32, 64]
    check(gpu_mx(x, splits), oracle.mx_group_cast(workloads.bits(x), splits), "special values K=416")


def test_graphsafe_unaligned_identical_and_tail_untouched():
    K, cap = 544, 768
    splits = [32, 0, 288, 96]  # 416 routed rows of 768
    w = workloads.random_case(118, K, splits, capacity=cap, dist="wide")
    x = w.x.cuda()
    fd, offs = abi.routing_tensors(splits, K)
    out = abi.alloc_mx_outputs(cap, K)
    for t in out.values():
        t.fill_(0xA5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.nvfp4_mx_group_cast_graphsafe(x, fd, offs, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    total = sum(splits)
    got = {k: v.cpu().numpy() for k, v in out.items()}
    cut = {"row_data": total, "row_scale": total, "col_data": total * K // 2, "col_scale": total * K // 32}
    head = {k: v[:cut[k]] for k, v in got.items()}
    check(head, gpu_mx(w.x[:total], splits), "graph-safe vs host-split")
    check(head, oracle.mx_group_cast(workloads.bits(w.x[:total]), splits), "graph-safe vs oracle")
    for k, v in got.items():
        assert np.all(v[cut[k]:] == 0xA5), k


def test_dequantize_bit_exact():
    w = workloads.random_case(107, 1024, [256, 128], dist="wide")
    want = oracle.mx_group_cast(workloads.bits(w.x), w.m_splits)
    R, K = w.x.shape
    out = torch.empty(R, K, device="cuda")
    abi.nvfp4_mx_dequantize(torch.from_numpy(want["row_data"]).cuda(), torch.from_numpy(want["row_scale"]).cuda(),
                            R, K, out)
    torch.cuda.synchronize()
    ref = oracle.mx_dequantize(want["row_data"], want["row_scale"], R, K)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    # colwise slice of group 1: rows = K, cols = m_1
    m = w.m_splits[1]
    cd = oracle.col_slice(want["col_data"], w.m_splits, K, 1, 2)
    cs = oracle.col_slice(want["col_scale"], w.m_splits, K, 1, 32)
    outc = torch.empty(K, m, device="cuda")
    abi.nvfp4_mx_dequantize(torch.from_numpy(np.ascontiguousarray(cd)).cuda(),
                            torch.from_numpy(np.ascontiguousarray(cs)).cuda(), K, m, outc)
    torch.cuda.synchronize()
    refc = oracle.mx_dequantize(cd, cs, K, m)
    assert np.array_equal(outc.cpu().numpy().view(np.uint32), refc.view(np.uint32))


@pytest.mark.slow
def test_full_size_deepseek_sampled_groups():
    w = workloads.config3()
    got = gpu_mx(w.x, w.m_splits)
    xb = workloads.bits(w.x)
    K = w.K
    offs = workloads.row_offsets(w.m_splits)
    live = sorted((m, g) for g, m in enumerate(w.m_splits) if m > 0)
    for _, g in (live[-1], live[len(live) // 2], live[0]):
        o, m = offs[g], w.m_splits[g]
        want = oracle.mx_group_cast(xb[o:o + m], [m])
        assert np.array_equal(got["row_data"][o:o + m], want["row_data"])
        assert np.array_equal(got["row_scale"][o:o + m], want["row_scale"])
        assert np.array_equal(got["col_data"][K * o // 2:K * (o + m) // 2], want["col_data"])
        assert np.array_equal(got["col_scale"][K * o // 32:K * (o + m) // 32], want["col_scale"])


def test_graphsafe_cuda_graph_replays():
    """Captured once, replayed after new routings are written to the device
    buffers: every replay equals the host-split cast of that routing."""
    w = workloads.config4(capacity=4096)
    x = w.x.cuda()
    cap, K = x.shape
    fd = torch.zeros(w.E, dtype=torch.int64, device="cuda")
    offs = torch.zeros(w.E + 1, dtype=torch.int64, device="cuda")
    out = abi.alloc_mx_outputs(cap, K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def set_routing(splits):
        f, o = abi.routing_tensors(splits, K)
        fd.copy_(f)
        offs.copy_(o)

    set_routing(w.routings[0])
    abi.nvfp4_mx_group_cast_graphsafe(x, fd, offs, out, st)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        abi.nvfp4_mx_group_cast_graphsafe(x, fd, offs, out, st)
    for splits in w.routings[:4]:
        set_routing(splits)
        graph.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        total = sum(splits)
        got = {k: v.cpu().numpy() for k, v in out.items()}
        cut = {"row_data": total, "row_scale": total, "col_data": total * K // 2, "col_scale": total * K // 32}
        check({k: v[:cut[k]] for k, v in got.items()}, gpu_mx(w.x[:total], splits), "replay")
