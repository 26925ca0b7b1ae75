"""iS-KV hot path on B200: block-incremental truncated SVD of KV streams plus decode attention
over the compressed history, served by hand-written sm_100a CUDA kernels behind a C ABI
(``include/iskv.h``, ``libiskv.so``).

``binding`` mirrors the C entry points one to one; ``cache.IsKVCache`` is a thin owner of a handle
that allocates caller-side buffers with torch. Importing the package loads ``libiskv.so`` and
raises if it has not been built.
"""
from .binding import *  # noqa: F401,F403
from .binding import IsKVError, LIB_PATH, check, lib  # noqa: F401


def __getattr__(name):
    if name == "IsKVCache":
        from .cache import IsKVCache
        return IsKVCache
    raise AttributeError(name)
