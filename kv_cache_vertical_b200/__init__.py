"""HyQuant hybrid-precision attention on B200 (sm_100a).

The compute lives in ``libhq.so`` (hand-written CUDA behind a C ABI, declared
in ``include/hq.h``); :mod:`kv_cache_vertical_b200.hq` is the thin ctypes
binding.  :mod:`kv_cache_vertical_b200.synth` draws seeded synthetic inputs.

The binding is imported lazily so that the input generator can be used
without the CUDA library; any use of an attention call loads ``libhq.so``
and raises if it has not been built.
"""
import importlib

__all__ = ["hq", "synth"]


def __getattr__(name):
    # submodules first: `from kv_cache_vertical_b200 import build` must work
    # before libhq.so exists (it is what builds it)
    if name in ("hq", "synth", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    mod = importlib.import_module(f"{__name__}.hq")
    try:
        return getattr(mod, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
