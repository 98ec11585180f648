"""The one-launch kernel's bounded waits give up cleanly and say so.

A cast item of nvfp4_group_quantize waits, with a bounded spin, until every
amax item of its group is published (TransformerEngine #3649, grouped
row-scaled NVFP4 cast, Description: the cast consumes the amax step's
vectors). The test build of the library (libnvfp4rs_test.so, compiled with
NVFP4_TEST_HOOKS) can start the kernel's item counter at position 1, so the
one amax item of a one-tile problem is never claimed and the cast item's wait
has nothing that could end it. The kernel must then give up within its bound
(about a second), record the give-up -- workspace word 1 for the host-split
call, NVFP4_ERR_TIMEOUT in the status word for the graph-safe one -- and
return, leaving the context usable: the next call, with the counter starting
at 0, must be byte-exact against the oracle. No fault, trap or hang is
involved; the wait simply runs out.
"""
import contextlib
import ctypes
import time

import pytest
import torch

from nvfp4_row_scaled_b200 import abi, workloads

from .helpers import assert_identical, oracle_cast

pytestmark = pytest.mark.gpu

K, SPLITS = 128, [128]  # one tile: amax item at position 0, its cast item at position 1
GIVE_UP_LIMIT_S = 30.0  # the kernel's own bounds end it in about a second


@pytest.fixture(scope="module")
def test_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_library, build_test_library
    build_library()
    path = build_test_library()
    abi.lib()
    return path


@contextlib.contextmanager
def hooked(path):
    """Route the binding through the test build for the duration."""
    saved_lib, saved_path = abi._lib, abi.LIB_PATH
    abi._lib, abi.LIB_PATH = None, path
    try:
        L = abi.lib()
        L.nvfp4_test_set_first_position.argtypes = [ctypes.c_uint8]
        L.nvfp4_test_set_first_position.restype = None
        yield L
    finally:
        L.nvfp4_test_set_first_position(0)
        abi._lib, abi.LIB_PATH = saved_lib, saved_path


def _results(out, ra, ca):
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["row_amax"], got["col_amax"] = ra.cpu().numpy(), ca.cpu().numpy()
    return got


def test_host_split_wait_gives_up_and_context_stays_usable(test_lib):
    w = workloads.random_case(61, K, SPLITS)
    x = w.x.cuda()
    R, E = x.shape[0], len(SPLITS)
    with hooked(test_lib) as L:
        ws = abi.alloc_workspace(0, E)
        ra, ca = abi.alloc_amax(R, K, E)
        out = abi.alloc_outputs(R, K, E)
        L.nvfp4_test_set_first_position(1)
        t0 = time.perf_counter()
        abi.nvfp4_group_quantize(x, SPLITS, ra, ca, out, ws)
        torch.cuda.synchronize()
        took = time.perf_counter() - t0
        assert took < GIVE_UP_LIMIT_S, f"the bounded wait took {took:.1f} s"
        assert int(ws[4:8].view(torch.int32).item()) != 0, "the give-up was not recorded"
        # the same call with the counter at 0 completes normally, bit-exact
        L.nvfp4_test_set_first_position(0)
        abi.nvfp4_group_quantize(x, SPLITS, ra, ca, out, ws)
        torch.cuda.synchronize()
        assert int(ws[4:8].view(torch.int32).item()) == 0
    assert_identical(_results(out, ra, ca), oracle_cast(w.x, SPLITS), what="after a give-up")


def test_graphsafe_wait_reports_timeout_status(test_lib):
    w = workloads.random_case(62, K, SPLITS)
    x = w.x.cuda()
    R, E = x.shape[0], len(SPLITS)
    fd, offs = abi.routing_tensors(SPLITS, K)
    with hooked(test_lib) as L:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = abi.alloc_workspace(R, E)
        ra, ca = abi.alloc_amax(R, K, E)
        out = abi.alloc_outputs(R, K, E)
        L.nvfp4_test_set_first_position(1)
        abi.nvfp4_group_quantize_graphsafe(x, fd, offs, ra, ca, out, ws, status)
        torch.cuda.synchronize()
        assert int(status.item()) == abi.NVFP4_ERR_TIMEOUT
        L.nvfp4_test_set_first_position(0)
        abi.nvfp4_group_quantize_graphsafe(x, fd, offs, ra, ca, out, ws, status)
        torch.cuda.synchronize()
        assert int(status.item()) == abi.NVFP4_OK
    assert_identical(_results(out, ra, ca), oracle_cast(w.x, SPLITS), what="graph-safe after a give-up")
