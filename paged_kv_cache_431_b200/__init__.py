"""Paged KV-cache attention for NVIDIA B200 (sm_100a).

The compute lives in ``libpkv.so`` (hand-written CUDA kernels behind a C-ABI,
declared in ``include/pkv.h``).  ``paged_kv_cache_431_b200.pkv`` is the thin Python
binding with the same entry-point names; ``workloads`` holds the seeded synthetic
inputs.  The binding is imported lazily so that the input generators can be used
without loading the CUDA library.
"""

__all__ = ["pkv", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
