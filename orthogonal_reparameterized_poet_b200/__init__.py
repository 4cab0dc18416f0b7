"""B200-native (sm_100a) hot path of the POET reparameterized linear layer.

The product is the C-ABI library ``libpoet.so`` (include/poet.h); ``poet`` is
its thin Python binding and ``inputs`` the seeded synthetic workloads.
Importing the package does not load the CUDA library; the first binding call
does, and raises if it is missing.
"""
__all__ = ["poet", "inputs"]
