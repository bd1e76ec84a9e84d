"""Fused Mixture-of-Experts layer for NVIDIA B200 (sm_100a).

The layer runs in libfused_moe.so (C ABI in include/fused_moe.h); `capi` is its
ctypes binding and `inputs` the seeded synthetic input generator.  `capi` is
imported lazily so that the input generator can be used without the library.
"""
import importlib

__all__ = ["capi", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
