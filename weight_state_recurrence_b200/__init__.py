"""B200-native causal linear attention as a fast-weight recurrence.

The compute lives in ``liblinattn.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/linattn.h``); :mod:`.linattn` is the thin ctypes
binding with the same entry-point names.  Importing the package does not load
the library; the first call does, and fails loudly if it is missing.
"""
__all__ = ["linattn", "inputs"]
