"""Writes the oracle-derived regression fixtures in this folder.

Calls only ``oracle/``; run from the repository root:
    python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402


def main():
    v64, v32 = oracle.codebook()
    with open(os.path.join(HERE, "nf4_codebook_reading.txt"), "w") as f:
        f.write("# NF4 levels under reading R1 (asymmetric normal quantiles, offset\n")
        f.write("# ((1-1/32)+(1-1/30))/2, divided by the largest). Written by make_golden.py from\n")
        f.write("# the oracle; a regression fixture for the reading, not a value printed on a page.\n")
        f.write("# index fp64 fp32_hex\n")
        for i in range(16):
            f.write(f"{i} {v64[i]:.17g} {np.float32(v32[i]).view(np.uint32):08x}\n")


if __name__ == "__main__":
    main()
