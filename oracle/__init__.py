"""Oracle for the QLoRA NF4 linear layer -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct CPU restatement of what the GPU library computes, in fp64 wherever the
method leaves the precision open.  It shares no code, table or constant with the CUDA library and imports
nothing from it.  Only the test suite, the package's ``smoke()`` check and the CPU-baseline leg of the
benchmark may import it; the product path never does.

Modules
-------
``oracle.nf4``     NF4 codebook, blockwise quantize / dequantize, bf16 round-to-nearest-even.
``oracle.linear``  forward / backward of the QLoRA linear layer, SwiGLU, and the gated-MLP chain.
``oracle.merge``   LoRA merge W' = deq(W) + s B A and its NF4 requantization.
``oracle.double_quant``  double quantization of the block constants (8-bit E4M3 codes, 256 per group).
``oracle.nvfp4``   the NVFP4 base-weight format: E2M1 codes, an E4M3 scale per 16, one fp32 scale per tensor.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against values fixed by the
mathematics (closed forms, invariants, brute force on tiny inputs, finite differences, library routines
for the special cases that reduce to them).  The exact NF4 table, which the pages name but do not print, is
pinned to the sixteen values printed in the paper that defines NF4 (QLoRA: Efficient Finetuning of Quantized
LLMs, Appendix E, "NormalFloat 4-bit data type"), kept as text in ``tests/golden/nf4_qlora_paper.txt`` and checked
by ``tests/test_oracle_nf4.py``.
"""

from . import nf4, linear, merge, double_quant, nvfp4  # noqa: F401
