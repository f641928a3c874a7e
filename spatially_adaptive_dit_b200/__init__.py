"""B200-native (sm_100a) mask-free spatially adaptive DiT attention path.

The compute lives in libsafedit.so (C ABI, include/safedit.h); the Python
binding is `spatially_adaptive_dit_b200.safedit`, which loads it and fails
loudly when it is missing.  `workloads` draws the seeded synthetic inputs.
"""
