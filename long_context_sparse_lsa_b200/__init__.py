"""B200-native (sm_100a) LongCat Sparse Attention hot path.

``binding`` wraps the C ABI of ``liblsa.so`` (include/lsa.h); it is imported
on first use of one of its names so that ``inputs`` and ``workloads`` stay
usable on a machine without the built library. Using a binding name without
the library raises immediately: there is no fallback implementation.
"""
from __future__ import annotations

_BINDING_NAMES = {
    "lsa_hi_block_sums", "lsa_append", "lsa_index", "lsa_attend", "lsa_attend_fp8", "lsa_index_workspace_size",
    "lsa_attend_workspace_size", "lsa_version", "Batch", "Budget", "LsaError", "library_path",
    "load_library",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
