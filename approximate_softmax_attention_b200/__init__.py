"""Approximate-softmax fused attention for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libqsm.so`` built from ``csrc/``
(TMA + tcgen05/TMEM kernels).  ``qsm`` is the thin ctypes binding with the
same entry-point names as ``include/qsm.h``; importing this package does not
load the library, calling an entry point does, and it raises if the library
is missing or no CUDA device is present (there is no CPU fallback).
"""

from . import inputs  # noqa: F401

__all__ = ["inputs", "qsm"]


def __getattr__(name):
    if name == "qsm":
        import importlib
        return importlib.import_module(__name__ + ".qsm")
    raise AttributeError(name)
