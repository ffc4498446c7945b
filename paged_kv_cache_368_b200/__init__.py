"""libpaged: PagedAttention decode and cache append for B200 (sm_100a).

The CUDA library ``libpaged.so`` (C ABI, header ``include/paged.h``) does the
work; :mod:`paged_kv_cache_368_b200.libpaged` is a thin ctypes binding over
it and is loaded on first use.  :mod:`paged_kv_cache_368_b200.inputs` makes
seeded synthetic workloads.
"""

__all__ = ["libpaged", "inputs"]


def __getattr__(name):
    if name in ("libpaged", "inputs"):
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
