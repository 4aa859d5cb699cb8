"""B200-native paged KV-cache decode path.

The CUDA library (``libpagedkv.so``, C ABI in ``include/pagedkv.h``) holds
the kernels; :mod:`paged_kv_cache_324_b200.binding` is a thin ctypes layer
over it that takes torch tensors.  Importing this package loads nothing: the
library is loaded on first use, and every call fails loudly if it is missing.
"""

__all__ = ["binding", "workload", "build"]
