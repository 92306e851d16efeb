"""B200-native (sm_100a) MoE expert layer: top-k routing or router replay,
stable dispatch, block-scaled FP8, grouped FP8 GEMMs on tcgen05, weighted
combine, and the backward.  The compute is in libmoe.so (C ABI, include/moe.h);
``abi`` binds it and ``layer`` sequences it.  ``inputs`` draws the seeded
synthetic workloads.
"""
__all__ = ["abi", "layer", "inputs", "build"]
