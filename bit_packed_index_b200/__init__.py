"""B200-native bit-packed VQ/RVQ linear layers.

The compute path is the C-ABI library ``libvq.so`` (hand-written sm_100a CUDA
kernels, declared in ``include/vq.h``); ``vq`` is its thin Python binding.
``bitrate`` is host-side size arithmetic.  Importing the package does not load
the CUDA library; the first call into ``vq`` does, and fails loudly if it is
missing.
"""
import importlib

__all__ = ["bitrate", "vq"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
