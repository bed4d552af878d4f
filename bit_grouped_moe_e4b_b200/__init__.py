"""Packed-4-bit Mixture-of-Experts layer for B200 (sm_100a).

The compute lives in the C-ABI library ``libe4b.so`` (``csrc/``, declared in
``include/e4b.h``); ``e4b`` is its thin ctypes binding. Importing this package
does not load the library; the first call into ``e4b`` does, and raises if the
library is missing. There is no CPU fallback.
"""

__all__ = ["configs", "synth", "e4b"]
