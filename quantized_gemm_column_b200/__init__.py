"""Averis mean-residual split NVFP4 linear layer on B200 (sm_100a).

The compute lives in ``libaveris.so`` (hand-written CUDA for sm_100a behind
a C ABI, declared in ``include/averis.h``); ``api`` is a thin ctypes binding
with the same entry-point names.  The library is loaded on first use and a
missing or unloadable library raises: there is no CPU fallback.
"""
