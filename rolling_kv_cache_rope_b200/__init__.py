"""B200-native rolling KV cache + fused 3D-RoPE attention (sm_100a).

The compute lives in ``librkv.so`` (CUDA kernels behind a C ABI declared in
``include/rkv.h``); ``rolling_kv_cache_rope_b200.rkv`` is a thin ctypes binding
with the same names.  Importing this package loads nothing; the first use of a
binding name loads the library and raises if it has not been built (there is no
CPU fallback).
"""

import importlib

_SUBMODULES = ("rkv", "synth", "build", "shard")
__all__ = list(_SUBMODULES)


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    if name in _SUBMODULES:
        return importlib.import_module(f"{__name__}.{name}")
    rkv = importlib.import_module(f"{__name__}.rkv")
    try:
        return getattr(rkv, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
