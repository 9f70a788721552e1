"""Regenerate the oracle regression fixture ``oracle_small_seeded.json``.

The stored values come from the fp64 oracle only (this script imports nothing
else that computes attention); the test suite uses them to notice any later
change in the oracle's arithmetic.  Inputs are drawn from numpy's seeded
generator and stored in the fixture verbatim.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(20240117)
    B, T, n_head, hs = 1, 6, 2, 4
    C = n_head * hs
    qkv = rng.standard_normal((B, T, 3 * C))
    dy = rng.standard_normal((B, T, C))
    y, lse = oracle.forward(qkv, n_head)
    dqkv = oracle.backward(qkv, dy, n_head)
    fx = {
        "note": "regression values written by tests/golden/make_golden.py from the fp64 oracle",
        "B": B, "T": T, "n_head": n_head, "head_size": hs,
        "qkv": qkv.tolist(), "dy": dy.tolist(),
        "y": y.tolist(), "lse": lse.tolist(), "dqkv": dqkv.tolist(),
    }
    with open(os.path.join(HERE, "oracle_small_seeded.json"), "w") as f:
        json.dump(fx, f, indent=0)


if __name__ == "__main__":
    main()
