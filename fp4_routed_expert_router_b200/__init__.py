"""Routed-expert FP4 FFN of a DeepSeek-V4.1-Flash-shaped MoE layer on B200.

The compute path lives in ``libmoe_fp4.so`` (hand-written CUDA for sm_100a
behind a C ABI, declared in ``include/moe_fp4.h``); ``moe`` is its thin ctypes
binding.  ``synth`` holds the seeded input generators.  Importing the package
does not load the CUDA library; ``moe.load()`` does, and fails loudly if it is
missing.
"""
__all__ = ["synth", "moe"]
