"""The GPU suite again, against the bounds-checked debug build.

libnvfp4rs_debug.so is the same library compiled with NVFP4_CHECK_BOUNDS:
every global store, atomic and explicit global load of every kernel checks
that it falls inside the buffers its call was given (sized from the call's
arguments), and counts -- instead of making -- any access outside them. This
test reruns the GPU tests in a child process with that build loaded
(NVFP4RS_LIBRARY); an autouse fixture there fails any test that leaves a
nonzero count. The outputs are the release build's: the checks only guard
accesses, they change no arithmetic, so the parity assertions apply as they
are.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# every GPU test file but this one and the timeout test (which loads the
# test-hook build itself)
SKIP = {"test_gpu_bounds.py", "test_gpu_timeout.py"}


def test_gpu_suite_under_the_bounds_checked_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_row_scaled_b200.build import build_debug_library
    lib = build_debug_library()
    files = sorted(f for f in os.listdir(os.path.join(ROOT, "tests"))
                   if (f.startswith("test_gpu_") or f.startswith("test_zz_")) and f.endswith(".py")
                   and f not in SKIP)
    env = dict(os.environ, NVFP4RS_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        *[os.path.join("tests", f) for f in files]],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).strip().splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
