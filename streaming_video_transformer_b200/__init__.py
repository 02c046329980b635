"""Streaming paged KV-cache attention for B200 (sm_100a).

The product is the C-ABI library ``libsvt.so`` (include/svt.h); this package
holds its CUDA sources (``csrc/``), the build step (``build.py``), a thin
ctypes binding (``cache.PagedKVCache``) and the seeded synthetic input
recipes (``inputs``).  Importing the package loads nothing; the binding
loads the library on first use and raises if it has not been built.
"""

__all__ = ["PagedKVCache", "SvtError"]


def __getattr__(name):
    if name in __all__:
        from . import cache
        return getattr(cache, name)
    raise AttributeError(name)
