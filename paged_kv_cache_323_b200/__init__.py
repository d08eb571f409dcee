"""B200-native paged KV-cache decode path.

The compute path is the C-ABI library ``libpagedkv.so`` (hand-written CUDA for
sm_100a, built from ``csrc/``); :mod:`paged_kv_cache_323_b200.pagedkv` is its
thin ctypes binding and raises on import when the library has not been built.
:mod:`paged_kv_cache_323_b200.workload` draws the seeded synthetic inputs.
"""
