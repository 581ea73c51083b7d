"""SVDQuant W4A4 + low-rank linear layer for B200 (sm_100a).

The compute lives in ``libsvdq.so`` (hand-written CUDA kernels behind the C
ABI declared in ``include/svdq.h``); ``bit_w4a4_quantized_b200.svdq`` is the
thin ctypes binding over it.  ``workloads`` holds the seeded input
generators.  Submodules are imported lazily so that the generators can be used
without loading the shared library.
"""

import importlib

__all__ = ["svdq", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
