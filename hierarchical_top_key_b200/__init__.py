"""B200-native HISA hierarchical indexer and flat DSA indexer.

The compute path lives in ``libhisa.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/hisa.h``).  ``binding`` marshals torch tensors into
that ABI; ``synthetic`` draws the seeded benchmark inputs.
"""
