"""Exact FlashAttention-2 forward and backward for B200 (sm_100a).

The compute path is the C-ABI library ``libfa2.so`` built from ``csrc/``
(declared in ``include/fa2.h``); ``fa2.py`` is its thin ctypes binding.  Importing
this package loads nothing: the library is opened on first use and a missing
library is an error, never a fallback.
"""
