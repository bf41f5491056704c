"""Writes nuq3_codebook.json: the eight fp16 centroids of the 3-bit non-uniform
datatype for keys and for values of the KVQuant-style workload.

Calls only the oracle (plain 1-D Lloyd k-means, oracle.nuq_fit) on a seeded sample of
the workload's synthetic keys and values (synth): the key vectors are channels over
128-token groups, the value vectors are token rows, each with its top-2 magnitudes
left out as outliers.  Run from the repository root:  python tests/golden/make_nuq3_codebook.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import nuq_fit  # noqa: E402


def main():
    cfg = synth.CONFIGS["kvquant_nuq3"]
    T = 2048
    kvec, vvec = [], []
    for h in range(4):
        K = synth.kv_slab(cfg, 0, h, T, "k").astype(np.float64)
        V = synth.kv_slab(cfg, 0, h, T, "v").astype(np.float64)
        for g0 in range(0, T, 128):
            kvec.extend(K[g0:g0 + 128].T)
        vvec.extend(V[:512])
    ck = nuq_fit.fit_codebook(np.array(kvec), 2)
    cv = nuq_fit.fit_codebook(np.array(vvec), 2)
    out = {
        "source": "oracle.nuq_fit.fit_codebook on synth kvquant_nuq3 (b=0, heads 0-3, "
                  "T=2048), 2 outliers per vector",
        "k": [float(x) for x in ck],
        "v": [float(x) for x in cv],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "nuq3_codebook.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)


if __name__ == "__main__":
    main()
