"""B200-native ResidualQuant hot path: KV-cache residual encode and fused
dequantise-and-reconstruct split-K decode attention for looped Transformers.

The compute lives in the C-ABI library ``librq_b200.so`` (hand-written CUDA for
sm_100a, built in-tree); ``rq`` is its thin ctypes binding.  Importing this
package does not load the library: ``from looped_transformer_decode_rq_b200
import rq`` does, and raises if the library has not been built.
"""
__all__ = ["rq", "synth"]
