"""Write tests/golden/tiny_oracle.npz from the CPU oracle alone.

The MoBiQuant explainer pages print no numeric worked example, so the stored
values here are the oracle's own outputs on the tiny seeded workload (N=256,
K=512, T=16, seed 0). They pin the oracle against silent drift: a later change
to its arithmetic must state the passage of the pages that justifies it.
Run: python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from token_adaptive_mixed_b200 import workloads as wl  # noqa: E402


def main():
    L = wl.tiny()
    codes, sz, _ = oracle.pack(L.W, S=3)
    k, gap, logits = oracle.route(L.X, L.Wr, L.bias)
    perm, off = oracle.bucket(k)
    Y = oracle.gemm(L.X, k, codes, sz, L.N)
    np.savez_compressed(os.path.join(HERE, "tiny_oracle.npz"), codes=codes, sz=sz, k_t=k, gap=gap,
                        perm=perm, offsets=off, Y=Y)


if __name__ == "__main__":
    main()
