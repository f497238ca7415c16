"""B200-native (sm_100a) hot path of the Wan2.1 / Wan2.2 video DiT.

The compute lives in the C-ABI library ``libwan.so`` (CUDA kernels for
sm_100a, declared in ``include/wan.h``); ``wan`` is its thin ctypes binding.
"""
