"""Writes ``oracle_small.json``: a small fixed case with the fp64 oracle's output.

The fixture is a regression record of the oracle (any later change to its
arithmetic shows up as a diff of this file). Inputs come from numpy's PCG64
generator with a fixed seed; the expected output comes from ``oracle/`` only.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import default  # noqa: E402


def case():
    rng = np.random.default_rng(20241014)
    B, N, H, d = 1, 6, 2, 4
    Q, K, V = (np.round(rng.standard_normal((B, N, H, d)), 3) for _ in range(3))
    Q[0, 2, 1, :] = -np.abs(Q[0, 2, 1, :]) - 0.5  # a phi(Q) = 0 row
    return Q, K, V, 1e-15


def main():
    Q, K, V, eps = case()
    orc = default()
    S = orc.state(K, V)
    O = orc.apply(Q, S, eps)
    doc = {
        "about": "ReLU linear attention forward, fp64 oracle output (regression record)",
        "shape_BNHd": list(Q.shape),
        "eps": eps,
        "Q": Q.ravel().tolist(), "K": K.ravel().tolist(), "V": V.ravel().tolist(),
        "state_BHd_dp1": S.ravel().tolist(),
        "O": O.ravel().tolist(),
    }
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
