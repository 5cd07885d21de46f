"""Exact scaled-dot-product attention for B200 (sm_100a).

The CUDA library ``libattn.so`` (built from ``csrc/``) exports the C ABI
declared in ``include/attn.h``; ``online_softmax_12_b200.attn`` is its thin
ctypes binding.  Importing the binding loads the library and raises if it is
missing: there is no fallback.  ``online_softmax_12_b200.inputs`` holds the
seeded synthetic input generators.
"""
__all__ = ["attn", "inputs"]
