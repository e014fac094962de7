"""Writes tiny_topk.json: small integer-valued indexer problems and the oracle's
Top-K for them.  Inputs are drawn here with numpy's seeded generator; expected
values come only from oracle/.  Re-run after a change to the oracle's
arithmetic that a passage of the pages justifies."""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import certified_topk, dense_topk  # noqa: E402


def main():
    rng = np.random.default_rng(2024)
    cases = []
    for T, S, H, d, K in [(6, 40, 3, 5, 4), (9, 70, 4, 6, 7), (5, 33, 2, 8, 40)]:
        q = rng.integers(-4, 4, (T, H, d))
        w = rng.integers(-4, 4, (T, H))
        k = rng.integers(-4, 4, (S, d))
        pos = np.sort(rng.choice(S, T, replace=False))
        dense = dense_topk(q.astype(float), w.astype(float), k.astype(float), pos, K)
        cert, tot = certified_topk(q.astype(float), w.astype(float), k.astype(float), pos, K,
                                   r=2, G=2, seed_first=4, seed_last=8, tile=8)
        cases.append({"q": q.tolist(), "w": w.tolist(), "k": k.tolist(), "positions": pos.tolist(),
                      "K": K, "dense_topk": dense.tolist(), "certified_topk": cert.tolist(),
                      "counts": tot})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_topk.json")
    with open(path, "w") as f:
        json.dump({"source": "tests/golden/make_golden.py (oracle/ only)", "cases": cases}, f)


if __name__ == "__main__":
    main()
