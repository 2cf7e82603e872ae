"""CPU oracle for paged KV-cache attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference arms may import this package.  The product path (the CUDA library
and its Python binding) never imports it, and the two share no code.
"""
from .pkv_oracle import *  # noqa: F401,F403
