"""B200-native decode hot path of Joint Subspace Sparse Attention (JSSA).

The compute lives in ``libjssa.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/jssa.h``).  This package is the thin Python binding:
``ops`` marshals torch CUDA tensors to that ABI; ``inputs`` draws the seeded
synthetic workloads; ``build`` compiles the library in-tree.  The library is
loaded on first use and a missing or unloadable library raises; there is no
fallback path.
"""
import importlib

__all__ = ["ops", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(__name__ + "." + name)
    raise AttributeError(name)
