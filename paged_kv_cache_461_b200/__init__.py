"""B200-native paged attention over a block-managed KV cache.

The compute path is the C-ABI library ``libpa_b200.so`` (hand-written CUDA for
sm_100a, declared in ``include/pa.h``).  ``paged_kv_cache_461_b200.api`` is a
thin ctypes binding with the same entry-point names; ``workloads`` builds
seeded synthetic inputs.  Importing the package loads nothing: the library is
opened on first use, and every call fails loudly if it is missing.
"""

__all__ = ["api", "workloads"]
