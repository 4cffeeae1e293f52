"""Exact fused attention forward and paged-KV decode for B200 (sm_100a).

The compute runs in hand-written CUDA kernels behind a C ABI
(``include/attn_b200.h``); :mod:`.api` is a thin ctypes binding over it that
takes torch CUDA tensors.  Importing this package does not load the CUDA
library; the first call into :mod:`.api` does, and raises if it is missing.
"""

import importlib

__all__ = ["api", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
