"""B200-native SparsePR per-call sparse attention.

The operator lives in the CUDA library ``libsparsepr.so`` (C ABI in include/sparsepr.h);
``native`` is its ctypes binding and ``workloads`` the seeded synthetic inputs.  The
library is loaded on first use, so importing the package needs no GPU.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads", "native"]


def __getattr__(name):
    if name == "native":
        import importlib
        return importlib.import_module(__name__ + ".native")
    raise AttributeError(name)
