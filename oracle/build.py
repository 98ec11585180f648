"""Compile the plain C oracle into ``libnvfp4_oracle.so`` next to this file.

Test infrastructure only (see ``nvfp4_oracle.h``). The flags keep every float
operation a single IEEE binary32 rounding: no contraction into FMA, no fast
math, SSE arithmetic on x86-64.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB = os.path.join(HERE, "libnvfp4_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard", "-Wall", "-Wextra"]


def build_oracle(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its sources."""
    srcs = [SRC, os.path.join(HERE, "nvfp4_oracle.h")]
    if not force and os.path.exists(LIB):
        if os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in srcs):
            return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force="--force" in sys.argv))
