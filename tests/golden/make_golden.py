"""Writes the stored expected values under tests/golden/ from the oracle alone.

    python tests/golden/make_golden.py

nf4_codebook.txt      the fp32 NF4 table built by oracle.nf4.nf4_codebook (normal-quantile rule, reading R1)
nf4_worked_block.txt  a hand-checkable block: w_j = c_(j mod 16) / 2 for j = 0..63, so absmax = 1/2 (the
                      level c_15 = 1 halves to 1/2), every quotient w_j / absmax is exactly c_(j mod 16), and
                      the codes are j mod 16, packed two per byte with element 2j in the high nibble.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import nf4 as O  # noqa: E402


def main():
    c = O.nf4_codebook()
    with open(os.path.join(HERE, "nf4_codebook.txt"), "w") as f:
        f.write("# NF4 codebook, fp32, ascending: index, bit pattern (hex), value\n")
        f.write("# written by tests/golden/make_golden.py from oracle.nf4.nf4_codebook\n")
        for i, v in enumerate(c):
            f.write(f"{i:2d} {int(v.view(np.uint32)):08x} {float(v):.9g}\n")
    w = np.array([c[j % 16] / np.float32(2) for j in range(64)], dtype=np.float32)
    codes, absmax = O.nf4_quantize(w)
    with open(os.path.join(HERE, "nf4_worked_block.txt"), "w") as f:
        f.write("# one 64-element block with w_j = c_(j mod 16) / 2; expected absmax and packed codes\n")
        f.write("# written by tests/golden/make_golden.py from oracle.nf4.nf4_quantize\n")
        f.write(f"absmax {int(absmax.view(np.uint32)[0]):08x}\n")
        hexs = codes.tobytes().hex()
        for k in range(0, len(hexs), 32):
            f.write(hexs[k:k + 32] + "\n")


if __name__ == "__main__":
    main()
