"""B200-native rolling KV cache + fused 3D-RoPE attention (sm_100a).

The compute lives in ``librkv.so`` (CUDA kernels behind a C ABI declared in
``include/rkv.h``); ``rolling_kv_cache_rope_b200.rkv`` is a thin ctypes binding
with the same names.  Importing this package loads nothing; the first use of a
binding name loads the library and raises if it has not been built (there is no
CPU fallback).
"""

__all__ = ["rkv", "synth"]


def __getattr__(name):
    if name == "rkv":
        from . import rkv
        return rkv
    if name == "synth":
        from . import synth
        return synth
    from . import rkv
    try:
        return getattr(rkv, name)
    except AttributeError:
        raise AttributeError(f"module 'rolling_kv_cache_rope_b200' has no attribute {name!r}") from None
