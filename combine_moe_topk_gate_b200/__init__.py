"""B200-native MoE routing: top-k gate, layout, dispatch and combine.

The compute path is the C-ABI library ``libmoe.so`` (hand-written sm_100a CUDA
kernels, declared in ``include/moe.h``).  :mod:`.api` is a thin ctypes binding
with the same names as the C entry points; it only marshals torch tensors
(device memory and streams) into pointers and sizes.  Importing :mod:`.api`
raises if the library has not been built: there is no fallback path.

:mod:`.workloads` (seeded synthetic inputs) does not need the library.
"""
from __future__ import annotations

import importlib

__all__ = ["api", "workloads"]


def __getattr__(name):
    if name in ("api", "workloads", "build"):
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
