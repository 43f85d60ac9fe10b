"""UFP4 4-bit training GEMMs for NVIDIA B200 (sm_100a).

The compute path lives in ``libufp4.so`` (CUDA, C ABI declared in
``include/ufp4.h``); :mod:`fp4_quantized_gemms_b200.ufp4` is a thin ctypes
binding over it.  The library is loaded on first use and every entry point
raises if it is missing or no CUDA device is present: there is no CPU path.
"""
__all__ = ["ufp4", "workloads", "recipe"]


def __getattr__(name):
    if name in ("ufp4", "recipe"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
