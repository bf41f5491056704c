"""Writes kqv_codebooks.json: the Lloyd-Max centroids of the coordinate marginal of a
uniformly random unit vector in R^128 (the KQV scheme's scalar codebook, after the
Walsh-Hadamard rotation), for 1 to 4 bits, as float64 and rounded to fp32.

Calls only the oracle (oracle.kqv.lloyd_max).  Run from the repository root:
    python tests/golden/make_kqv_codebooks.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import kqv  # noqa: E402

D = 128


def codebooks():
    return {str(b): [float(x) for x in kqv.lloyd_max(b, D)] for b in (1, 2, 3, 4)}


def main():
    cb = codebooks()
    out = {
        "source": "oracle.kqv.lloyd_max(bits, d=128), bits 1..4",
        "d": D,
        "f64": cb,
        "f32": {b: [float(np.float32(x)) for x in v] for b, v in cb.items()},
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "kqv_codebooks.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
