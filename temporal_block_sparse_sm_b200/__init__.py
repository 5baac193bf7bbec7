"""B200-native LiteAttention: temporally sparse attention with a persistent skip mask.

The compute path is the CUDA library ``libliteattn.so`` (sm_100a), reached
through the ctypes binding in :mod:`temporal_block_sparse_sm_b200.liteattn`.
Importing this package does not load the library; the first call that needs
it does, and raises if it is missing.
"""
__all__ = ["liteattn", "synthetic"]
