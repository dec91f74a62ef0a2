"""Causal sliding-window attention for B200 (sm_100a).

The compute lives in the C-ABI library ``libswa_b200.so`` (hand-written CUDA
kernels, declared in ``include/swa_attn.h``). ``causal_sliding_window_b200.ops``
is the thin ctypes binding with the same entry-point names; importing it loads
the library and raises if it is missing. ``inputs`` holds the seeded synthetic
input generators and never loads the library.
"""
import importlib

__all__ = ["ops", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
