"""SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).

The compute lives in libsvdq.so (C ABI: include/svdq.h), built in-tree by
``python -m rank_gemm_b200.build``.  ``rank_gemm_b200.binding`` is the thin
ctypes layer over it; its names are re-exported here on first use, and
importing them fails loudly if the library has not been built.
"""
import importlib

__all__ = ["binding", "build"]


def __getattr__(name):
    if name in ("build",):
        return importlib.import_module(".build", __name__)
    mod = importlib.import_module(".binding", __name__)
    if name == "binding":
        return mod
    return getattr(mod, name)
