"""B200-native (sm_100a) block-sparse decode attention for Elastic Threshold
Attention (ETA).

The decode path runs entirely in ``libeta.so`` (CUDA kernels behind the C ABI
of ``include/eta.h``); :mod:`learned_block_sparse_b200.binding` is its thin
ctypes binding. Importing :mod:`binding` fails loudly if the library is absent.
"""
__all__ = ["binding", "synth"]
