"""B200-native predict-then-quantize-residual KV-cache codec.

The compute path is the C-ABI library ``libkvc.so`` (hand-written sm_100a CUDA
kernels); ``clustered_kv_cache_b200.kvc`` is its thin ctypes binding.  Importing
this package does not load the library; the first call into ``kvc`` does, and
raises if it is missing.  ``synth`` holds the seeded synthetic workloads.
"""
