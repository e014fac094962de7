"""Pins of the oracle's ranked threshold schedule and of the ideal prune count.

The ranked schedule screens every non-warm-up key once against an estimate of
the threshold, then checks the estimate with the exact K-th it reached (a
further passes over bands of lower bounds when a key it rejected is not
below it).  The pins: its
selection is the dense one (brute-force definition), every key it rejects
scores strictly below the true K-th, and it never rejects more than the ideal
screening (threshold equal to the true K-th) would.  The ideal count itself is
pinned where the bound has a closed form (UB = I)."""
import numpy as np
import pytest

from oracle import (certificate_setup, certified_topk_row, dense_topk, indexer_scores,
                    key_mean, ranked_topk_row, seed_mask, soundness_margin, upper_bound)


def _instance(rng, T=10, H=12, d=16, S=900, redundant=False):
    if redundant:
        base = rng.standard_normal((T, 1, d))
        q = base + 0.05 * rng.standard_normal((T, H, d))
        w = np.abs(rng.standard_normal((T, H))) / 8
        w[:, ::4] *= -1
    else:
        q = 0.8 * rng.standard_normal(d) + rng.standard_normal((T, H, d))
        w = rng.standard_normal((T, H)) / 8
    k = rng.standard_normal((S, d)) + 0.3
    k[::53] *= 4.0
    return q, w, k


@pytest.mark.parametrize("redundant", [False, True])
@pytest.mark.parametrize("r,G,K,warm,spread", [(4, 2, 8, 3, 2.0), (2, 1, 30, 2, 1.0),
                                                (0, 0, 5, 4, 2.0), (4, 2, 64, 2, 0.25),
                                                (4, 0, 20, 6, 8.0)])
def test_ranked_selection_is_dense_and_rejections_are_sound(redundant, r, G, K, warm, spread):
    rng = np.random.default_rng(K * 7 + r + warm + int(redundant))
    q, w, k = _instance(rng, redundant=redundant)
    T, S = q.shape[0], k.shape[0]
    pos = np.linspace(40, S - 1, T).astype(int)
    kb = key_mean(k)
    want = dense_topk(q, w, k, pos, K)
    for t in range(T):
        kv = k[: pos[t] + 1]
        res = ranked_topk_row(q[t], w[t], kv, K, k_bar=kb, warm_tiles=warm, r=r, G=G,
                              seed_first=8, seed_last=32, tile=16, spread=spread)
        assert np.array_equal(res["idx"], want[t])
        I = indexer_scores(q[t], w[t].astype(np.float64), kv)
        rej = ~res["exact_mask"]
        assert np.all(I[rej] < res["v_K"])           # nothing rejected could tie the K-th
        assert res["tau"] <= res["v_K"]
        assert res["rejected"] <= res["ideal_rejected"]
        # the ideal count can never exceed the keys that score below the K-th
        screened = ~seed_mask(pos[t], 8, 32) & ~(np.arange(pos[t] + 1) < 16)
        assert res["ideal_rejected"] <= int(np.sum(screened & (I < res["v_K"])))


def test_ranked_later_passes_recover_an_estimate_set_too_high():
    """m = 1: the first estimate is the largest warm-up score, far above the
    K-th, so pass 1 keeps too few keys; the later passes (lower estimates, the
    last one the warm-up's own K-th) must restore the exact result while still
    rejecting most keys."""
    rng = np.random.default_rng(3)
    q, w, k = _instance(rng, T=4, S=1200, redundant=True)
    kb = key_mean(k)
    for t in range(4):
        res = ranked_topk_row(q[t], w[t], k, 40, k_bar=kb, warm_tiles=3, seed_first=8,
                              seed_last=32, tile=16, spread=1e-6)
        assert res["m"] == 1
        assert res["passes"] >= 2
        assert np.diff(res["estimates"]).max() <= 0 and res["estimates"][-1] <= res["v_K"]
        assert res["rejected"] > 0.5 * res["visible"]
        assert np.array_equal(res["idx"], dense_topk(q[t:t + 1], w[t:t + 1], k,
                                                     np.array([k.shape[0] - 1]), 40)[0])


def test_ranked_schedule_reaches_the_ideal_on_redundant_heads():
    """Near-copy heads: the bound is tight and the estimate lands a little
    below the K-th, so over the rows the ranked schedule rejects nearly all
    the ideal screening (threshold = the true K-th) does, in one pass."""
    rng = np.random.default_rng(11)
    q, w, k = _instance(rng, T=8, S=6000, redundant=True)
    kb = key_mean(k)
    got = ideal = 0
    for t in range(8):
        res = ranked_topk_row(q[t], w[t], k, 64, k_bar=kb, warm_tiles=20, seed_first=8,
                              seed_last=32, tile=16)
        got += res["rejected"]
        ideal += res["ideal_rejected"]
        assert res["passes"] == 1
    assert got >= 0.93 * ideal
    assert ideal > 0.85 * 8 * 6000


def test_ideal_rejected_in_the_closed_form_where_the_bound_is_the_score():
    """Every positive head retained (r = |P|) and every negative head in one
    group active on every key: UB = I, so the ideal count is exactly the
    non-seed keys whose score plus margin is below the true K-th."""
    rng = np.random.default_rng(21)
    H, d, n, K = 6, 8, 600, 12
    k_dir = rng.standard_normal(d)
    q_t = rng.standard_normal((H, d)) * 0.2 + k_dir
    w_t = np.array([0.3, -0.2, 0.5, -0.1, 0.4, -0.25])
    k = k_dir + 0.3 * rng.standard_normal((n, d))
    assert np.all(k @ q_t.T > 0)
    P = int((w_t > 0).sum())
    cert = certificate_setup(q_t, w_t, key_mean(k), P, 1)
    np.testing.assert_allclose(upper_bound(cert, q_t, k), indexer_scores(q_t, w_t, k),
                               rtol=1e-12, atol=1e-12)
    I = indexer_scores(q_t, w_t, k)
    vK = np.sort(I)[-K]
    delta = soundness_margin(q_t, w_t, k, -12)
    seeds = seed_mask(n - 1, 8, 32)
    want = int(np.sum(~seeds & (I + delta < vK)))
    res = certified_topk_row(q_t, w_t, k, K, k_bar=key_mean(k), r=P, G=1, seed_first=8,
                             seed_last=32, tile=16)
    assert res["ideal_rejected"] == want
    assert want > n // 2


def test_stored_prune_study_matches_a_fresh_oracle_run():
    """tests/golden/prune_study.json is written by tests/prune_study.py from
    the oracle alone (64 rows per workload).  A fresh run of the same code on
    one row per workload must agree with its conclusions: at the library's
    head budget (r = 4) the mandated generator leaves nothing to prune, even
    every positive head retained leaves the negative aggregate loose, and
    redundant heads prune most pairs."""
    import json
    import os
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, here)
    import prune_study
    with open(os.path.join(here, "golden", "prune_study.json")) as f:
        stored = {r["workload"]: r for r in json.load(f)["results"]}
    assert stored["prefill_128k_fp8"]["ideal_prune_pct"]["r=4,G=2"] < 0.01
    assert stored["tight_64k_bf16_levels"]["ideal_prune_pct"]["r=4,G=2"] < 0.01
    assert stored["redundant_chunk128k_fp8"]["ideal_prune_pct"]["r=4,G=2"] > 90.0
    assert len(stored["prefill_128k_fp8"]["rows"]) == 64
    from dataclasses import replace
    from exact_certified_top_b200.workloads import WORKLOADS, generate, small_case, codes_numpy
    from oracle import dequantize, key_mean
    for name, lo, hi in (("prefill_128k_fp8", 0.0, 0.01), ("redundant_chunk128k_fp8", 50.0, 100.0)):
        wl = small_case(name, 2, 16384, q_pos0=16382)
        x = generate(wl)
        ks = None if x["k_scale"] is None else x["k_scale"].numpy()
        k = dequantize(codes_numpy(x["k"]), ks, wl.dtype)
        qs = None if x["q_scale"] is None else x["q_scale"][1:2].numpy()
        q = dequantize(codes_numpy(x["q"][1:2]), qs, wl.dtype)[0]
        res = prune_study.row_study(q, x["w"][1].numpy().astype(np.float64),
                                    k[: wl.q_pos0 + 2], key_mean(k), wl.K)
        pct = 100.0 * res["ideal"]["r=4,G=2"] / res["visible"]
        assert lo <= pct <= hi, (name, pct)
        assert res["ranked_rejected"] <= res["ideal"]["r=4,G=2"]
