"""Regenerate the oracle regression fixtures ``oracle_small_seeded.json`` and
``block_small_seeded.json`` (the attention sub-block oracle).

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
import oracle.block as block  # noqa: E402


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

    # the pre-LN attention sub-block on a small seeded input
    B, T, C, n_head = 1, 5, 8, 2
    x = rng.standard_normal((B, T, C)) * 1.5 + 0.3
    p = {"ln_w": 1.0 + 0.2 * rng.standard_normal(C), "ln_b": 0.1 * rng.standard_normal(C),
         "w_attn": rng.standard_normal((3 * C, C)) / np.sqrt(C), "b_attn": 0.1 * rng.standard_normal(3 * C),
         "w_proj": rng.standard_normal((C, C)) / np.sqrt(C), "b_proj": 0.1 * rng.standard_normal(C)}
    out, qkv_b, y_b, lse_b = block.attn_block_forward(x, n_head=n_head, attention=oracle.forward, **p)
    fb = {"note": "regression values written by tests/golden/make_golden.py from the block oracle",
          "B": B, "T": T, "C": C, "n_head": n_head, "x": x.tolist(), **{k: v.tolist() for k, v in p.items()},
          "out": out.tolist(), "qkv": qkv_b.tolist(), "y": y_b.tolist(), "lse": lse_b.tolist()}
    with open(os.path.join(HERE, "block_small_seeded.json"), "w") as f:
        json.dump(fb, f, indent=0)


if __name__ == "__main__":
    main()
