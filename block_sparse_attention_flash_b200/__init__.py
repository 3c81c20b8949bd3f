"""Block-sparse softmax attention for video DiTs on B200 (sm_100a).

The compute path is the C-ABI library ``libsparse_attn.so`` built from
``csrc/``; ``ops`` is a thin ctypes binding over it (argument marshalling
only).  ``inputs`` holds the seeded synthetic workload generators.
"""
__all__ = ["inputs", "ops"]
