"""B200-native low-rank binary factorised linear: y = s1 * (U (V^T (s2 * x))).

The compute lives in the CUDA C-ABI library ``libnq.so`` (declared in ``include/nq.h``);
``binary_rank_linear_02_b200.nq`` is its thin ctypes binding.  The binding is imported
lazily so that ``synth`` (seeded inputs) can be used on machines without the library.
"""
from __future__ import annotations

import importlib

__all__ = ["nq", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
