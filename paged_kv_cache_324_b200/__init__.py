"""B200-native paged KV cache: decode and chunked-prefill attention over a
block-table-addressed pool, the scatter, copy-on-write and swap kernels, and a
native block manager with prefix caching.

The CUDA library (``libpagedkv.so``, C ABI in ``include/pagedkv.h``) holds
the kernels and the block manager; :mod:`paged_kv_cache_324_b200.binding` is a thin ctypes layer
over it that takes torch tensors.  Importing this package loads nothing: the
library is loaded on first use, and every call fails loudly if it is missing.
"""

__all__ = ["binding", "workload", "build"]
