"""QLoRA NF4 linear layer for B200 (sm_100a): blockwise NF4 base weight + bf16 LoRA, forward and backward.

The compute runs in the CUDA library ``libqlora.so`` (built from ``csrc/``) behind a C ABI declared in
``include/qlora.h``; ``qlora_fine_tuning_blockwise_b200.ops`` is the thin Python binding over it.
Importing this package does not load the library; the first call into ``ops`` does, and fails loudly
if the library is missing.
"""

__all__ = ["inputs", "ops"]
