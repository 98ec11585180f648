"""Build ``libnvfp4rs.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

The library is one translation unit (``csrc/nvfp4rs.cu``) compiled with
IEEE-exact float settings: no FMA contraction, IEEE divides, no flush to zero,
so that the device arithmetic is the one the header documents.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libnvfp4rs.so")
# the same library with -DNVFP4_TEST_HOOKS, loaded only by the timeout test
TEST_LIB = os.path.join(HERE, "libnvfp4rs_test.so")
# the bounds-checked debug build (-DNVFP4_CHECK_BOUNDS, see csrc/bounds.cuh)
DEBUG_LIB = os.path.join(HERE, "libnvfp4rs_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "--fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
    "--cudart", "static",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))] + [
        os.path.join(INCLUDE, "nvfp4rs.h")]


def _build(lib: str, extra, force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib):
        if os.path.getmtime(lib) >= max(os.path.getmtime(s) for s in sources()):
            return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "nvfp4rs.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than any source."""
    return _build(LIB, [], force, verbose)


def build_test_library(force: bool = False) -> str:
    """The library with its test hooks (see NVFP4_TEST_HOOKS in nvfp4rs.cu)."""
    return _build(TEST_LIB, ["-DNVFP4_TEST_HOOKS"], force, False)


def build_debug_library(force: bool = False) -> str:
    """The bounds-checked debug build: every global access of the kernels is
    checked against the ranges registered for its launch."""
    return _build(DEBUG_LIB, ["-DNVFP4_CHECK_BOUNDS"], force, False)


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_test_library(force="--force" in sys.argv))
    print(build_debug_library(force="--force" in sys.argv))
