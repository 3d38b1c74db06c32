"""B200-native B-spline Kolmogorov-Arnold (KAN) layer: forward and backward.

The compute lives in ``libkan_b200.so`` (hand-written sm_100a CUDA behind a C
ABI, ``include/kan_b200.h``).  ``_native`` is its ctypes binding with the same
names; ``layer`` holds the torch-facing calls and the drop-in ``KANLayer``.
Importing the package does not load the library; the first compute call does,
and fails loudly if it is missing.
"""
from . import workloads  # noqa: F401  (no native code)

__all__ = ["forward", "backward", "basis", "KANLayer", "KANNetwork", "workloads"]


def __getattr__(name):
    if name in ("forward", "backward", "basis", "KANLayer", "KANNetwork", "workspace", "shape_of"):
        from . import layer
        return getattr(layer, name)
    raise AttributeError(name)
