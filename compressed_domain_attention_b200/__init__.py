"""B200-native rotation-based int4 KV-cache quantisation and compressed-domain decode attention.

The compute path is the C-ABI shared library ``libtq_b200.so`` (CUDA kernels
for sm_100a, declared in ``include/tq.h``); ``tq`` is its thin ctypes binding.
Importing this package does not load the library; the first call into ``tq``
does, and raises if it is missing (there is no CPU fallback).
"""

__all__ = ["tq", "synthetic"]
