"""B200-native KDA (Kimi Delta Attention) recurrence: chunked prefill with KCP
inter-chunk state composition, and single-token decode.

The compute path is ``libkda.so`` (hand-written sm_100a CUDA kernels behind a
C ABI declared in ``include/kda.h``); ``kda`` is its thin Python binding and
``inputs`` the seeded synthetic-input generator. Importing the binding raises
if the shared library has not been built: there is no CPU fallback.
"""
import importlib

__all__ = ["kda", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
