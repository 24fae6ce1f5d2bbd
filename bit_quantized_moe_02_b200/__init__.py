"""2-bit block-quantized routed-MoE FFN on NVIDIA B200 (sm_100a).

The compute path lives in the C-ABI library ``libds4moe.so`` (hand-written
CUDA, see ``csrc/``); ``bit_quantized_moe_02_b200.ds4moe`` is its ctypes
binding.  ``bit_quantized_moe_02_b200.synth`` holds the seeded synthetic input
generators.  Importing this package loads nothing; the binding loads the
library on first use and raises if it is missing.
"""
__all__ = ["synth", "ds4moe"]
