"""Writes the oracle's 8-bit (256-level) Lloyd-Max codebooks for the widths
the GPU parity tests quantise at, so that those tests need not re-solve them
(the oracle takes one to two minutes per 8-bit codebook).  It calls only the
oracle (oracle.codebook); each file holds the centroids and then the
thresholds, one float.hex() per line.

    python tests/golden/make_oracle_codebooks.py
"""
import os
import sys
from concurrent.futures import ProcessPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
WIDTHS = (1536, 3072, 4096, 12288)
BITS = 8


def path(d, bits):
    return os.path.join(HERE, f"oracle_codebook_d{d}_b{bits}.txt")


def write(d):
    sys.path.insert(0, ROOT)
    import oracle

    c, t = oracle.codebook(d, BITS)
    with open(path(d, BITS), "w") as f:
        f.write(f"# oracle.codebook({d}, {BITS}): {len(c)} centroids then {len(t)} thresholds, float.hex\n")
        for v in list(c) + list(t):
            f.write(float(v).hex() + "\n")
    return d


if __name__ == "__main__":
    with ProcessPoolExecutor(max_workers=len(WIDTHS)) as ex:
        for d in ex.map(write, WIDTHS):
            print("wrote", path(d, BITS))
