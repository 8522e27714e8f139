"""B200-native token-pruned attention for video diffusion transformers.

The compute path lives in ``libtps.so`` (hand-written sm_100a CUDA behind a C
ABI, header ``include/tps.h``); ``token_pruned_sparse_b200.tps`` is the thin
ctypes binding. ``synth`` makes seeded synthetic inputs.
"""
__version__ = "0.1.0"
