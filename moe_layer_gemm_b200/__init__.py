"""B200-native forward pass of one Mixture-of-Experts FFN layer.

The compute lives in a C-ABI shared library of hand-written sm_100a CUDA
kernels (``lib/libmoe_b200.so``); this package is its thin ctypes binding
(``moe_layer_gemm_b200.abi``) plus seeded synthetic workloads
(``moe_layer_gemm_b200.synth``).  Importing the package does not load the
library; the first call into ``abi`` does, and fails loudly if it is missing.
"""
__all__ = ["abi", "synth"]
