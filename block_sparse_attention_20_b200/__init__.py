"""B200-native AB-Attention hot path (IBCS selector, SIP sampler, gather attention).

The compute lives in ``libabatt.so`` (CUDA, sm_100a) behind the C ABI declared
in ``include/abatt.h``; :mod:`.abatt` is the thin ctypes binding.  Importing
this package does not load the library; the first call does, and raises if
it is missing.
"""
