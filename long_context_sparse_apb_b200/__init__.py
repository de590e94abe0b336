"""APB per-host prefill path on B200: retaining-head scoring and top-k
compression, passing-block construction and block-masked attention, run as
hand-written sm_100a CUDA kernels behind the C ABI declared in include/apb.h.

``inputs`` (workload configurations and seeded synthetic data) imports
without the CUDA library; the kernels are reached through ``apb``, which loads
the in-tree shared library and raises if it is missing.
"""
import importlib

__all__ = ["inputs", "apb"]


def __getattr__(name):
    if name == "apb":
        return importlib.import_module(__name__ + "._lib")
    if name == "inputs":
        return importlib.import_module(__name__ + ".inputs")
    raise AttributeError(name)
