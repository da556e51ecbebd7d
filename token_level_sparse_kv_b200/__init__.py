"""B200-native decode hot path of Joint Subspace Sparse Attention (JSSA).

The compute lives in ``libjssa.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/jssa.h``).  This package is the thin Python binding:
``ops`` marshals torch CUDA tensors to that ABI; ``inputs`` draws the seeded
synthetic workloads.  The library is loaded on first use and a missing or
unloadable library raises; there is no fallback path.
"""
__all__ = ["ops", "inputs"]


def __getattr__(name):
    if name == "ops":
        from . import ops as _ops

        return _ops
    if name == "inputs":
        from . import inputs as _inputs

        return _inputs
    raise AttributeError(name)
