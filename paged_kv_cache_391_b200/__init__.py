"""B200-native paged-KV-cache decode: the PagedAttention hot path.

The compute lives in ``libpa.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/pa.h``). ``paged_kv_cache_391_b200.pa`` is the thin
ctypes binding; ``paged_kv_cache_391_b200.workloads`` builds seeded inputs.
Importing this package loads nothing: the library is opened on first use and
a missing library is an error, never a fallback.
"""
__all__ = ["pa", "workloads"]


def __getattr__(name):
    if name in ("pa", "workloads"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
