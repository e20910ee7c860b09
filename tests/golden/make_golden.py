"""Writes the stored expected values under tests/golden/ by calling only the oracle.

  nf4_codebook.txt   the 16-entry NF4 codebook as binary16 bit patterns.

The pages name the NF4 codebook ("deep-fold", section "Method": each group of
64 weights stores four-bit NF4 codes and one FP16 scale) but never print its
values, so the table is built by the oracle's NormalFloat construction
(sixteen normal quantiles, 8 positive, 7 negative, an exact zero, scaled to
[-1, 1]) and rounded to binary16.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def main():
    cb = oracle.nf4_codebook()
    vals = oracle.h2f(cb)
    path = os.path.join(HERE, "nf4_codebook.txt")
    with open(path, "w") as fh:
        fh.write("# NF4 codebook, binary16 bit patterns in increasing order, one per line.\n")
        fh.write("# Source: the NF4 (NormalFloat) data type named on the \"deep-fold\" page,\n")
        fh.write("# section \"Method\"; the page prints no values.  Written by\n")
        fh.write("# tests/golden/make_golden.py from the oracle's construction.\n")
        for i, (b, v) in enumerate(zip(cb, vals)):
            fh.write(f"0x{int(b):04x}  # {i:2d}: {float(v):+.8f}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
