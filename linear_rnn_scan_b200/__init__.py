"""B200-native MRU prefix-product scan.

The compute path is the CUDA library ``libmru.so`` (sm_100a kernels behind a
C-ABI declared in ``include/mru.h``); ``linear_rnn_scan_b200.mru`` is a thin
ctypes binding with the same entry-point names.  ``inputs`` holds the seeded
synthetic input generators.  Importing the package loads nothing; the binding
loads the library on first use and raises if it has not been built.
"""
from __future__ import annotations

import importlib

__all__ = ["mru", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
