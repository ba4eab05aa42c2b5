"""B200-native DiT-MoE sparse expert layer (forward, with the balance loss's
statistics and gradient): C-ABI library + thin binding.

``inputs`` (seeded synthetic workloads) and ``metrics`` (work accounting) load
without a GPU.  The compute entry points live in ``binding`` (ctypes over
``libmoe.so``) and ``layer`` (buffer management around the four calls); they
load the CUDA library on import and fail loudly when it is missing.
"""
import importlib

__all__ = ["inputs", "metrics", "binding", "layer"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
