"""B200 (sm_100a) MoE expert-parallel dispatch / combine over W virtual ranks.

The compute lives in libep_b200.so (C ABI: include/ep.h); ``binding`` is its
ctypes binding. Names of the binding are re-exported here on first use; that
import fails loudly when the library has not been built (``build`` builds it).
"""
import importlib


def __getattr__(name):
    if name.startswith("__") or name in ("build", "binding"):
        raise AttributeError(name)
    return getattr(importlib.import_module(__name__ + ".binding"), name)
