"""Pins of the oracle's dense indexer: the score definition and the Top-K rule.

Each pin checks the oracle against something other than itself: pure-Python
brute force, hand-computed closed forms, exact integer arithmetic, and an
independent selection by repeated argmax."""
import itertools
import random

import numpy as np
import pytest

from oracle import dense_topk, indexer_scores, select_topk


def brute_scores(q_t, w_t, k):
    """Pure-Python loops, no numpy arithmetic."""
    out = []
    for ks in k.tolist():
        tot = 0.0
        for qh, wh in zip(q_t.tolist(), w_t.tolist()):
            dot = sum(a * b for a, b in zip(qh, ks))
            tot += wh * (dot if dot > 0 else 0.0)
        out.append(tot)
    return out


def argmax_select(scores, K):
    """Independent selection: repeatedly take the largest remaining score,
    smallest index first on ties."""
    remaining = list(range(len(scores)))
    chosen = []
    for _ in range(min(K, len(scores))):
        best = remaining[0]
        for s in remaining[1:]:
            if scores[s] > scores[best]:
                best = s
        chosen.append(best)
        remaining.remove(best)
    return sorted(chosen) + [-1] * (K - len(chosen))


def test_hand_example_relu_sign_and_ties():
    # x_0 = q_0.k = [1, 2, 0, -3], x_1 = q_1.k = [-1, 1, -3, 0]
    # I = 0.5*ReLU(x_0) - 2*ReLU(x_1) = [0.5, -1, 0, 0]
    q_t = np.array([[1.0, 2.0], [-1.0, 1.0]])
    w_t = np.array([0.5, -2.0])
    k = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, -1.0], [-1.0, -1.0]])
    assert indexer_scores(q_t, w_t, k).tolist() == [0.5, -1.0, 0.0, 0.0]
    # keys 2 and 3 tie at 0: the smaller index wins
    assert select_topk(indexer_scores(q_t, w_t, k), 2).tolist() == [0, 2]
    assert select_topk(indexer_scores(q_t, w_t, k), 3).tolist() == [0, 2, 3]
    # fewer keys than K: all of them, then -1
    assert select_topk(indexer_scores(q_t, w_t, k), 6).tolist() == [0, 1, 2, 3, -1, -1]


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    H, d, n = rng.integers(1, 5), rng.integers(1, 9), rng.integers(1, 40)
    q_t = rng.standard_normal((H, d))
    w_t = rng.standard_normal(H)
    k = rng.standard_normal((n, d))
    got = indexer_scores(q_t, w_t, k)
    want = brute_scores(q_t, w_t, k)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    for K in (1, 3, 8, n, n + 5):
        assert select_topk(got, K).tolist() == argmax_select(want, K)


def test_integer_inputs_are_exact():
    """Small integers: every score is an integer computed exactly, so the oracle
    must equal Python's exact integer arithmetic bit for bit."""
    rng = random.Random(3)
    H, d, n = 5, 7, 50
    q_t = [[rng.randint(-4, 3) for _ in range(d)] for _ in range(H)]
    w_t = [rng.randint(-4, 3) for _ in range(H)]
    k = [[rng.randint(-4, 3) for _ in range(d)] for _ in range(n)]
    exact = [sum(w * max(0, sum(a * b for a, b in zip(qh, ks))) for qh, w in zip(q_t, w_t))
             for ks in k]
    got = indexer_scores(np.array(q_t, float), np.array(w_t, float), np.array(k, float))
    assert got.tolist() == [float(v) for v in exact]
    # integer scores tie often; ranking by (score desc, index asc) with Python's sort
    ranked = sorted(range(n), key=lambda s: (-exact[s], s))
    assert select_topk(got, 11).tolist() == sorted(ranked[:11])


def test_single_head_unit_weight_reduces_to_relu_dot_topk():
    """H = 1, w = 1: the score is ReLU(q.k); the Top-K must equal the K largest of
    ReLU(q.k) by a library partial sort on (-score, index)."""
    rng = np.random.default_rng(7)
    q_t = rng.standard_normal((1, 16))
    k = rng.standard_normal((300, 16))
    s = np.maximum(k @ q_t[0], 0.0)                 # many exact zeros: ties
    keys = np.array([(-v, i) for i, v in enumerate(s)], dtype=[("a", float), ("b", int)])
    part = np.sort(np.partition(keys, 40, order=["a", "b"])[:40], order=["a", "b"])
    assert select_topk(indexer_scores(q_t, np.ones(1), k), 40).tolist() == sorted(part["b"].tolist())


def test_causal_visibility_inclusive():
    """Row t sees keys 0..p_t inclusive: a dominant key at s = p_t is selected,
    one at s = p_t + 1 is not."""
    H, d, S = 2, 4, 10
    q = np.ones((3, H, d))
    w = np.ones((3, H))
    k = np.full((S, d), 0.1)
    k[5] = 10.0        # visible to the row at position 5
    k[6] = 100.0       # invisible to it
    out = dense_topk(q, w, k, positions=np.array([5, 6, 9]), K=1)
    assert out[:, 0].tolist() == [5, 6, 6]


def test_dense_rows_subset_matches_full():
    rng = np.random.default_rng(11)
    T, H, d = 20, 3, 5
    q = rng.standard_normal((T, H, d))
    w = rng.standard_normal((T, H))
    k = rng.standard_normal((T, d))
    pos = np.arange(T)
    full = dense_topk(q, w, k, pos, K=4)
    sub = dense_topk(q, w, k, pos, K=4, rows=[3, 17])
    assert np.array_equal(full[[3, 17]], sub)
    for t in range(T):
        want = argmax_select(brute_scores(q[t], w[t], k[: t + 1]), 4)
        assert full[t].tolist() == want


def test_negative_zero_ties_with_zero():
    scores = np.array([-0.0, 0.0, -0.0, -1.0])
    assert select_topk(scores, 2).tolist() == [0, 1]
