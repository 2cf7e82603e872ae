"""Paged KV-cache attention for B200 (sm_100a).

The compute path is the native library ``libpkv.so`` (hand-written CUDA behind
a C ABI, declared in ``include/pkv.h``).  This package is its thin Python
binding: it marshals torch tensors into pointers and sizes and raises when the
library reports an error.  Importing a binding name loads the library and
fails loudly if it has not been built; there is no fallback path.

``workloads`` (seeded synthetic inputs) imports without the library.
"""
from importlib import import_module

_API = (
    "PkvError", "Cache", "Plan", "kv_append", "plan_attention", "paged_attention", "split_kv_reduce",
    "attention_workspace_bytes", "default_num_ctas", "library_path", "status_string", "DTYPE_CODES",
    "GraphStep", "paged_attention_noalloc",
)

__all__ = list(_API) + ["workloads"]


def __getattr__(name):
    if name in _API:
        return getattr(import_module(".api", __name__), name)
    if name == "workloads":
        return import_module(".workloads", __name__)
    raise AttributeError(name)
