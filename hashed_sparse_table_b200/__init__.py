"""B200 (sm_100a) hot path of the Memory Layer trainable in-model embedding cache.

``binding`` is the ctypes binding of ``libmpzch.so`` (the CUDA kernels);
``inputs`` draws the seeded synthetic workloads.  ``binding`` is imported on
first use so that the input generator works on hosts without the built
library; using any table call without the library raises ImportError.
"""
import importlib

__all__ = ["binding", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
