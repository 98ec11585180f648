"""Consumer side of the cast on the GPU.

- Scales in the 128x4-tiled layout that block-scaled grouped GEMMs read (the
  swizzle contract of the grouped-experts four-over-six converter, torchtitan
  #14, Design notes): emitted by the cast itself, byte for byte the oracle's
  tiling of the oracle's compact scales; every other output unchanged; the
  host-split, graph-safe and one-launch calls agree; groups that are not
  multiples of 128 rows are refused.
- The FP32 per-row post-scale after a GEMM run with amax = 1
  (TransformerEngine #2931, sequence diagram): bit-exact against the oracle,
  f32 and bf16, with and without bias, in place; and end to end, a GEMM on
  the amax = 1 dequantization followed by the post-scale agrees with the GEMM
  on the true dequantization.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import KEYS, assert_identical, oracle_cast

pytestmark = pytest.mark.gpu

TILED = abi.NVFP4_SCALE_TILED_128X4


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library
    build_library()
    abi.lib()


def cast(x, splits, layout, path="two"):
    xd = x.cuda()
    R, K = xd.shape
    E = len(splits)
    ra, ca = abi.alloc_amax(R, K, E)
    out = abi.alloc_outputs(R, K, E)
    for t in out.values():
        t.view(torch.uint8).fill_(0xA5)
    if path == "two":
        abi.nvfp4_group_amax(xd, splits, ra, ca)
        abi.nvfp4_group_cast(xd, splits, ra, ca, out, scale_layout=layout)
    elif path == "graphsafe":
        fd, offs = abi.routing_tensors(splits, K)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        abi.nvfp4_group_amax_graphsafe(xd, fd, offs, ra, ca, st)
        abi.nvfp4_group_cast_graphsafe(xd, fd, offs, ra, ca, out, st, scale_layout=layout)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
    elif path == "one":
        abi.nvfp4_group_quantize(xd, splits, ra, ca, out, abi.alloc_workspace(0, E), scale_layout=layout)
    elif path == "noalloc":
        abi.nvfp4_group_quantize_noalloc(xd, splits, ra, ca, out, scale_layout=layout)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("K,splits,seed", [
    (512, [128, 256, 0, 384], 80),
    (256, [0, 128, 0, 0, 256, 128], 81),
    (7168, [256, 0, 128], 82),
])
def test_tiled_scales_against_oracle(K, splits, seed):
    w = workloads.random_case(seed, K, splits, dist="wide")
    want = oracle_cast(w.x, splits)
    tiled = oracle.swizzle_cast_scales(want, splits, K)
    got = cast(w.x, splits, TILED)
    assert_identical(got, {**want, **tiled}, keys=list(KEYS), what=f"K={K} {splits}")


@pytest.mark.parametrize("path", ["graphsafe", "one", "noalloc"])
def test_tiled_scales_every_path_agrees(path):
    w = workloads.config1()
    want = cast(w.x, w.m_splits, TILED, "two")
    assert_identical(cast(w.x, w.m_splits, TILED, path), want, keys=list(KEYS), what=path)


def test_tiled_scales_need_128_row_groups():
    K = 256
    splits = [48, 208]
    x = torch.zeros(256, K, dtype=torch.bfloat16, device="cuda")
    ra, ca = abi.alloc_amax(256, K, 2)
    out = abi.alloc_outputs(256, K, 2)
    abi.nvfp4_group_amax(x, splits, ra, ca)
    with pytest.raises(abi.NVFP4Error) as e:
        abi.nvfp4_group_cast(x, splits, ra, ca, out, scale_layout=TILED)
    assert e.value.status == abi.NVFP4_ERR_UNSUPPORTED
    fd, offs = abi.routing_tensors(splits, K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.nvfp4_group_cast_graphsafe(x, fd, offs, ra, ca, out, st, scale_layout=TILED)
    torch.cuda.synchronize()
    assert int(st.item()) == abi.NVFP4_ERR_UNSUPPORTED


@pytest.mark.slow
def test_tiled_scales_full_size_deepseek():
    """DeepSeek-V3 shape: the tiled scales are the oracle's tiling of the
    compact scales of the same call (those are checked against the oracle
    in test_gpu_fullsize), and every other output is unchanged."""
    w = workloads.config3()
    compact = cast(w.x, w.m_splits, abi.NVFP4_SCALE_COMPACT)
    tiled = cast(w.x, w.m_splits, TILED)
    want = oracle.swizzle_cast_scales(compact, w.m_splits, w.K)
    assert_identical(tiled, {**compact, **want}, keys=list(KEYS), what="deepseek tiled")


# ------------------------------------------------------------- post-scale

@pytest.mark.parametrize("rows,cols,bias,dtype", [
    (1, 4, False, torch.float32),
    (37, 132, True, torch.float32),
    (1000, 1028, False, torch.bfloat16),
    (513, 2048, True, torch.bfloat16),
])
def test_post_scale_against_oracle(rows, cols, bias, dtype):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    x = torch.randn(rows, cols, generator=g) * torch.exp2(torch.randint(-20, 20, (rows, 1), generator=g).float())
    a = torch.rand(rows, generator=g) * 100.0
    a[::7] = 0.0
    b = torch.randn(cols, generator=g) if bias else None
    wf, wb = oracle.row_post_scale(x.numpy(), a.numpy(), None if b is None else b.numpy())
    out = torch.empty(rows, cols, dtype=dtype, device="cuda")
    abi.nvfp4_row_post_scale(x.cuda(), a.cuda(), out, None if b is None else b.cuda())
    torch.cuda.synchronize()
    if dtype == torch.float32:
        assert np.array_equal(out.cpu().numpy().view(np.uint32), wf.view(np.uint32))
    else:
        assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), wb)


def test_post_scale_in_place_and_checks():
    g = torch.Generator().manual_seed(9)
    x = torch.randn(64, 256, generator=g)
    a = torch.rand(64, generator=g)
    wf, _ = oracle.row_post_scale(x.numpy(), a.numpy())
    xd = x.cuda()
    abi.nvfp4_row_post_scale(xd, a.cuda(), xd)
    torch.cuda.synchronize()
    assert np.array_equal(xd.cpu().numpy().view(np.uint32), wf.view(np.uint32))
    with pytest.raises(abi.NVFP4Error) as e:
        abi.nvfp4_row_post_scale(torch.zeros(4, 6, device="cuda"), torch.ones(4, device="cuda"),
                                 torch.zeros(4, 6, device="cuda"))
    assert e.value.status == abi.NVFP4_ERR_UNSUPPORTED


def test_gemm_with_unit_amax_then_post_scale_matches_true_dequant():
    """The fprop path of the pages: GEMM on the row-scaled operand decoded
    with amax = 1, rows multiplied back by the row amax, equals (to float
    rounding) the GEMM on the true decode."""
    w = workloads.random_case(90, 1024, [256, 128, 128], dist="wide")
    x = w.x.cuda()
    M, K = x.shape
    ra, ca = abi.alloc_amax(M, K, 3)
    out = abi.alloc_outputs(M, K, 3, col=False)
    abi.nvfp4_group_amax(x, w.m_splits, ra, None)
    abi.nvfp4_group_cast(x, w.m_splits, ra, None, out)
    true = torch.empty(M, K, device="cuda")
    abi.nvfp4_dequantize(out["row_data"], out["row_scale"], out["row_s2"], M, K, true)
    unit_s2 = torch.full((M,), float(oracle.s_dec(1.0)), device="cuda")
    unit = torch.empty(M, K, device="cuda")
    abi.nvfp4_dequantize(out["row_data"], out["row_scale"], unit_s2, M, K, unit)
    g = torch.Generator(device="cuda").manual_seed(4)
    Wt = torch.randn(K, 512, device="cuda", generator=g)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        y_true = true @ Wt
        y_unit = unit @ Wt
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    y = torch.empty_like(y_unit)
    abi.nvfp4_row_post_scale(y_unit, ra, y)
    torch.cuda.synchronize()
    scale = y_true.abs().amax(dim=1, keepdim=True).clamp_min(1e-30)
    assert float(((y - y_true).abs() / scale).max()) < 1e-5


def test_tiled_scales_graphsafe_cuda_graph_replays():
    w = workloads.config4(capacity=4096)
    x = w.x.cuda()
    cap, K = x.shape
    E = w.E
    fd = torch.zeros(E, dtype=torch.int64, device="cuda")
    offs = torch.zeros(E + 1, dtype=torch.int64, device="cuda")
    ra, ca = abi.alloc_amax(cap, K, E)
    out = abi.alloc_outputs(cap, K, E)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run():
        abi.nvfp4_group_amax_graphsafe(x, fd, offs, ra, ca, st)
        abi.nvfp4_group_cast_graphsafe(x, fd, offs, ra, ca, out, st, scale_layout=TILED)

    def set_routing(splits):
        f, o = abi.routing_tensors(splits, K)
        fd.copy_(f)
        offs.copy_(o)

    set_routing(w.routings[0])
    run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    for splits in w.routings[:4]:
        set_routing(splits)
        graph.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        total = sum(splits)
        got = {k: v.cpu().numpy() for k, v in out.items()}
        cut = {"row_data": total, "row_scale": total, "row_s2": total,
               "col_data": total * K // 2, "col_scale": total * K // 16}
        got = {k: (v[:cut[k]] if k in cut else v) for k, v in got.items()}
        assert_identical(got, cast(w.x[:total], splits, TILED), keys=list(KEYS), what="tiled replay")
