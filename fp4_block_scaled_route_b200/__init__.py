"""B200-native decode-regime MoE layer (FP8 / MXFP4 block-scaled experts).

The compute path is the CUDA library ``libmoe.so`` built from ``csrc/`` for
sm_100a; :mod:`fp4_block_scaled_route_b200.moe` is its thin ctypes binding
(argument marshalling only).  :mod:`fp4_block_scaled_route_b200.synth` holds
the seeded synthetic input generators.
"""

__all__ = ["moe", "synth"]
