"""Regression pin: the oracle reproduces its stored outputs on integer inputs
(exact arithmetic, so equality is bit for bit), and the certified and dense
selections agree on them."""
import json
import os

import numpy as np

from oracle import certified_topk, dense_topk

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_golden_cases():
    with open(os.path.join(HERE, "golden", "tiny_topk.json")) as f:
        data = json.load(f)
    for c in data["cases"]:
        q, w, k = (np.array(c[n], float) for n in ("q", "w", "k"))
        pos = np.array(c["positions"])
        dense = dense_topk(q, w, k, pos, c["K"])
        assert dense.tolist() == c["dense_topk"]
        cert, tot = certified_topk(q, w, k, pos, c["K"], r=2, G=2, seed_first=4, seed_last=8,
                                   tile=8)
        assert cert.tolist() == c["certified_topk"] == c["dense_topk"]
        assert tot == c["counts"]
