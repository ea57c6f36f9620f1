"""B200-native Lighthouse selection-and-attend layer (pool, score, top-K, gather + causal attention,
scatter-back; forward and backward) behind the C-ABI library ``liblh.so``.

The compute path is hand-written sm_100a CUDA; ``lh`` is a thin ctypes binding that only marshals arguments.
Importing ``lh`` fails loudly when the library has not been built.
"""

__all__ = ["lh", "inputs"]
