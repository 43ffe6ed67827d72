"""Writes tests/golden/tiny_d4_s6_t3.json from the float64 oracle (and nothing else).

Run from the repository root: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import gdn_scan_ref  # noqa: E402


def main():
    rng = np.random.default_rng(2024)
    T, S, D = 3, 6, 4
    # Dyadic inputs (multiples of 1/8) so the fixture's inputs are exact in any float type.
    q, k, v = (np.round(rng.standard_normal((T, S, D)) * 8) / 8 for _ in range(3))
    gamma = np.array([0.875, 0.96875, 0.9375])
    beta = np.array([0.5, 0.25, 0.75])
    m0 = np.round(rng.standard_normal((D, D)) * 8) / 8
    o, m = gdn_scan_ref(q, k, v, gamma, beta, state_in=m0)
    fx = {
        "what": "oracle output on a tiny dyadic case (regression fixture; written by make_golden.py)",
        "inputs": {"q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "gamma": gamma.tolist(),
                   "beta": beta.tolist(), "state_in": m0.tolist()},
        "out": o.tolist(),
        "state_out": m.tolist(),
    }
    with open(os.path.join(HERE, "tiny_d4_s6_t3.json"), "w") as f:
        json.dump(fx, f, indent=1)


if __name__ == "__main__":
    main()
