"""B200-native SVG-EAR clustered block-sparse attention.

The hot path (k-means, permutation, error probe, routing, block-sparse
attention with linear compensation) runs in libear.so, hand-written CUDA for
sm_100a behind the C ABI in include/ear.h.  ``clustered_block_sparse_b200.ear``
is the Python binding; ``inputs`` holds the seeded synthetic workloads.
"""
__all__ = ["ear", "inputs"]
