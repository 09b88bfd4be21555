"""B200-native MoE expert-parallel dispatch and combine.

The compute path is the CUDA library ``libep_b200.so`` (sm_100a) behind the C
ABI declared in ``include/ep.h``; ``combine_ep_dispatch_03_b200.ep`` is its
thin ctypes binding. Importing this package does not load the library; the
first call into ``ep`` does, and raises if it is missing.
"""
__version__ = "0.1.0"
