"""The oracle's codebooks stored under tests/golden by
tests/golden/make_oracle_codebooks.py (which calls only oracle.codebook), for
widths whose 8-bit solve takes the oracle minutes."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def stored_oracle_codebook(d, bits):
    """(centroids, thresholds) in fp64 as oracle.codebook returns them, from
    the stored file; solved by the oracle when no file is stored."""
    path = os.path.join(GOLDEN, f"oracle_codebook_d{d}_b{bits}.txt")
    if not os.path.exists(path):
        return oracle.codebook(d, bits)
    with open(path) as f:
        vals = [float.fromhex(ln.strip()) for ln in f if ln.strip() and not ln.startswith("#")]
    L = 1 << bits
    assert len(vals) == 2 * L - 1, (d, bits, len(vals))
    return np.array(vals[:L]), np.array(vals[L:])
