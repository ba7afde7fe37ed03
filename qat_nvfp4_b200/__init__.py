"""NVFP4 two-level block quantization and QAT fake-quantization for B200 (sm_100a).

The compute lives in ``libnvfp4.so`` (hand-written CUDA behind the C ABI declared in
``include/nvfp4.h``); :mod:`qat_nvfp4_b200.nvfp4` is the thin ctypes binding to it and
raises at import if the library has not been built.  :mod:`qat_nvfp4_b200.synthetic`
holds the seeded input generators.
"""
import importlib

__all__ = ["nvfp4", "synthetic"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module("." + name, __name__)
    binding = importlib.import_module(".nvfp4", __name__)
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
