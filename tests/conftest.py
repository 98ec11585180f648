import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size cases")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.lib()


@pytest.fixture(autouse=True)
def bounds_faults_stay_zero(request):
    """With the bounds-checked debug build loaded (NVFP4RS_LIBRARY), every GPU
    test must end with no access counted outside its launch's ranges."""
    if request.node.get_closest_marker("gpu") is None or "NVFP4RS_LIBRARY" not in os.environ:
        yield
        return
    from nvfp4_row_scaled_b200 import abi
    L = abi.lib()
    if not hasattr(L, "nvfp4_debug_bounds_faults"):
        yield
        return
    import ctypes
    L.nvfp4_debug_bounds_faults.restype = ctypes.c_ulonglong
    L.nvfp4_debug_bounds_reset()
    yield
    import torch
    torch.cuda.synchronize()
    faults = int(L.nvfp4_debug_bounds_faults())
    assert faults == 0, f"{faults} accesses outside their launch's registered ranges"
