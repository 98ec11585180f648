"""Grouped row-scaled (per-token) NVFP4 cast for B200 (sm_100a).

The compute lives in ``libnvfp4rs.so`` (hand-written CUDA behind a C ABI,
declared in ``include/nvfp4rs.h``); ``nvfp4_row_scaled_b200.abi`` is the thin
ctypes binding. Importing this package loads nothing: the library is opened on
the first call, and a call fails loudly if it is missing.
"""

__all__ = ["abi", "workloads"]
