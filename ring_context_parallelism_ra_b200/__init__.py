"""Ring Attention hot path for one B200 (sm_100a).

The compute lives in ``libra.so`` (hand-written CUDA behind a C ABI declared in
``include/ra.h``); ``ring_context_parallelism_ra_b200.ra`` is the thin ctypes
binding with the same entry-point names.  Importing this package does not load
the library; the first call into ``ra`` does, and raises if it is missing.
"""
__all__ = ["ra", "workloads"]
