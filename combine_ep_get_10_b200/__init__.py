"""B200-native MoE token layout / dispatch / combine (token choice and
expert choice).

The compute lives in ``libep_b200.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/ep.h``); ``binding`` is its thin ctypes binding
with the same entry-point names.  The library is loaded on first use and a
missing or unloadable library raises immediately: there is no fallback.
"""
import importlib

from .workloads import BF16, FP32, FP8_E4M3, COMPACT, PADDED  # noqa: F401


def __getattr__(name):
    if name == "binding" or name.startswith("ep_"):
        mod = importlib.import_module(__name__ + ".binding")
        return mod if name == "binding" else getattr(mod, name)
    raise AttributeError(name)
