"""Pins of the oracle's certificate: NNLS, bound soundness, closed-form
reductions, the seed threshold and the exactness of the certified selection."""
import itertools

import numpy as np
import pytest

from oracle import (certificate_setup, certified_topk, certified_topk_row, dense_topk,
                    indexer_scores, key_mean, nnls_retained, seed_mask, soundness_margin,
                    upper_bound)


def test_nnls_matches_grid_search_r2():
    rng = np.random.default_rng(0)
    for _ in range(20):
        Q = rng.standard_normal((2, 6))
        v = rng.standard_normal(6) + 0.5 * Q[0]
        a = nnls_retained(Q, v)
        assert np.all(a >= 0)
        grid = np.linspace(0, 3, 601)
        A0, A1 = np.meshgrid(grid, grid, indexing="ij")
        res = v[None, None, :] - A0[..., None] * Q[0] - A1[..., None] * Q[1]
        best = float(np.min(np.sum(res ** 2, axis=-1)))
        got = np.sum((v - a @ Q) ** 2)
        assert got <= best + 1e-9
        assert got >= best - 0.05      # the grid is fine enough to come close


@pytest.mark.parametrize("seed", range(5))
def test_nnls_kkt_r4(seed):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((4, 12)) + 1.0
    v = rng.standard_normal(12) + 1.0
    a = nnls_retained(Q, v)
    g = Q @ (v - a @ Q)            # minus the gradient of the objective / 2
    assert np.all(a >= 0)
    for j in range(4):
        if a[j] > 1e-12:
            assert abs(g[j]) < 1e-8    # stationary on the support
        else:
            assert g[j] <= 1e-8        # no descent direction off the support


@pytest.mark.parametrize("seed", range(4))
def test_nnls_library_solver_agrees_with_exhaustive_supports(seed):
    """The r > 4 path (scipy's active-set NNLS) against the exhaustive-support
    solver on r <= 4, and the KKT conditions at r = 8 and 16."""
    from scipy.optimize import nnls
    rng = np.random.default_rng(40 + seed)
    for r in (2, 3, 4):
        Q = rng.standard_normal((r, 10)) + 0.5
        v = rng.standard_normal(10) + 0.5
        a_lib, _ = nnls(Q.T, v)
        np.testing.assert_allclose(nnls_retained(Q, v), a_lib, atol=1e-9)
    for r in (8, 16):
        Q = rng.standard_normal((r, 32)) + 0.3
        v = rng.standard_normal(32) + 0.3
        a = nnls_retained(Q, v)
        g = Q @ (v - a @ Q)
        assert np.all(a >= 0)
        assert np.all(np.abs(g[a > 1e-10]) < 1e-8) and np.all(g[a <= 1e-10] <= 1e-8)


def test_nnls_exact_member_and_negative_target():
    Q = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 0.0]])
    assert np.allclose(nnls_retained(Q, np.array([2.0, 3.0, 5.0])), [2.0, 3.0])
    assert np.allclose(nnls_retained(Q, np.array([-2.0, 3.0, 0.0])), [0.0, 3.0])
    assert np.allclose(nnls_retained(Q, np.array([-2.0, -3.0, 1.0])), [0.0, 0.0])


def _instance(rng, H=16, d=24, n=400, corr=0.6):
    base = rng.standard_normal(d)
    q_t = corr * base + rng.standard_normal((H, d))
    w_t = rng.standard_normal(H) / 8
    k = 0.5 * rng.standard_normal(d) + rng.standard_normal((n, d))
    k[::37] *= 4.0
    return q_t, w_t, k


@pytest.mark.parametrize("r,G", [(0, 0), (1, 1), (2, 2), (4, 1), (4, 2), (8, 2)])
def test_upper_bound_dominates_score(r, G):
    rng = np.random.default_rng(r * 10 + G)
    for _ in range(4):
        q_t, w_t, k = _instance(rng)
        cert = certificate_setup(q_t, w_t, key_mean(k), r, G)
        # adversarial keys: along residual-heavy and head directions
        extra = np.vstack([q_t, -q_t, cert.u if cert.u.size else np.zeros((0, q_t.shape[1]))])
        kk = np.vstack([k, extra, 3 * extra])
        ub = upper_bound(cert, q_t, kk)
        I = indexer_scores(q_t, w_t, kk)
        assert np.all(ub >= I - 1e-9 * (1 + np.abs(I)))


def test_reduction_all_positive_retained_single_active_group_is_exact():
    """r = |P| and every negative head in one group that is active on the key:
    UB equals the score (closed form)."""
    rng = np.random.default_rng(5)
    H, d = 6, 8
    k_dir = rng.standard_normal(d)
    q_t = rng.standard_normal((H, d)) * 0.2 + k_dir      # every head active on k_dir
    w_t = np.array([0.3, -0.2, 0.5, -0.1, 0.4, -0.25])
    P = int((w_t > 0).sum())
    cert = certificate_setup(q_t, w_t, k_dir, r=P, G=1)
    assert cert.beta == 0.0 and len(cert.groups) == 1 and cert.groups[0].size == 3
    k = k_dir + 0.05 * rng.standard_normal((50, d))
    assert np.all(k @ q_t.T > 0)
    np.testing.assert_allclose(upper_bound(cert, q_t, k), indexer_scores(q_t, w_t, k),
                               rtol=1e-12, atol=1e-12)


def test_reduction_no_retained_no_groups_is_cauchy_schwarz():
    """r = 0, G = 0: UB = beta ||k|| with beta = min(sum w||q||, joint)."""
    rng = np.random.default_rng(6)
    q_t, w_t, k = _instance(rng, H=8, d=10, n=30)
    cert = certificate_setup(q_t, w_t, key_mean(k), r=0, G=0)
    P = w_t > 0
    assert np.isclose(cert.beta_sum, np.sum(w_t[P] * np.linalg.norm(q_t[P], axis=1)))
    Ws = np.sqrt(w_t[P])[:, None] * q_t[P]
    assert np.isclose(cert.beta_joint,
                      np.sqrt(w_t[P].sum() * np.linalg.eigvalsh(Ws.T @ Ws)[-1]))
    np.testing.assert_allclose(upper_bound(cert, q_t, k),
                               min(cert.beta_sum, cert.beta_joint) * np.linalg.norm(k, axis=1))


def test_two_negative_groups_never_looser_than_one():
    rng = np.random.default_rng(8)
    q_t, w_t, k = _instance(rng)
    c1 = certificate_setup(q_t, w_t, key_mean(k), 4, 1)
    c2 = certificate_setup(q_t, w_t, key_mean(k), 4, 2)
    c0 = certificate_setup(q_t, w_t, key_mean(k), 4, 0)
    u0, u1, u2 = (upper_bound(c, q_t, k) for c in (c0, c1, c2))
    assert np.all(u1 <= u0 + 1e-12) and np.all(u2 <= u1 + 1e-12)


def test_seed_mask():
    m = seed_mask(1000, 64, 512)
    assert m.sum() == 64 + 512 and m[:64].all() and m[489:].all() and not m[64:489].any()
    assert seed_mask(100, 64, 512).all()


def test_margin_scales_with_key_norm():
    q_t = np.array([[3.0, 4.0], [0.0, 1.0]])
    w_t = np.array([2.0, -1.0])
    k = np.array([[1.0, 0.0], [0.0, 2.0]])
    np.testing.assert_allclose(soundness_margin(q_t, w_t, k, -3), [11 / 8, 22 / 8])


@pytest.mark.parametrize("r,G,K", [(4, 2, 8), (2, 1, 30), (0, 0, 5), (4, 0, 64)])
def test_certified_selection_equals_dense_and_tau_is_lower_bound(r, G, K):
    rng = np.random.default_rng(K + r)
    T, H, d, S = 12, 12, 16, 700
    q = 0.8 * rng.standard_normal(d) + rng.standard_normal((T, H, d))
    w = rng.standard_normal((T, H)) / 8
    k = rng.standard_normal((S, d)) + 0.3
    pos = np.linspace(0, S - 1, T).astype(int)
    kb = key_mean(k)
    got, tot = certified_topk(q, w, k, pos, K, r=r, G=G, seed_first=8, seed_last=32, k_bar=kb)
    assert np.array_equal(got, dense_topk(q, w, k, pos, K))
    for t in range(T):
        res = certified_topk_row(q[t], w[t], k[: pos[t] + 1], K, k_bar=kb, r=r, G=G,
                                 seed_first=8, seed_last=32)
        assert res["tau0"] <= res["v_K"]
        assert res["tau_final"] <= res["v_K"]
        # the schedule's threshold never exceeds the true K-th, so it rejects a
        # subset of what the ideal threshold would reject
        assert res["rejected"] <= res["ideal_rejected"]
    assert tot["visible"] == int(np.sum(pos + 1))


def test_certified_prunes_when_heads_are_redundant():
    """A case the certificate is built for: identical positive heads and a
    clear winner set, so most keys are rejected."""
    rng = np.random.default_rng(9)
    H, d, S, K = 8, 16, 4000, 16
    base = rng.standard_normal(d)
    q_t = np.tile(base, (H, 1))
    w_t = np.abs(rng.standard_normal(H)) / 8
    k = rng.standard_normal((S, d))
    res = certified_topk_row(q_t, w_t, k, K, k_bar=key_mean(k), r=2, G=2,
                             seed_first=8, seed_last=32)
    assert np.array_equal(res["idx"], dense_topk(q_t[None], w_t[None], k, np.array([S - 1]), K)[0])
    assert res["rejected"] > 0.8 * res["visible"]


@pytest.mark.parametrize("r,G", [(0, 0), (2, 1), (4, 2)])
def test_block_bound_dominates_every_key_of_the_block(r, G):
    """UB_B >= UB(s) >= I(s) for every key of the block, including keys on the
    ball's boundary along the head and aggregate directions (where the
    per-key bound is largest)."""
    from oracle import block_upper_bound, key_block_stats
    rng = np.random.default_rng(100 + r * 10 + G)
    for _ in range(6):
        q_t, w_t, k = _instance(rng)
        cert = certificate_setup(q_t, w_t, key_mean(k), r, G)
        center = rng.standard_normal(q_t.shape[1])
        block = center + 0.3 * rng.standard_normal((128, q_t.shape[1]))
        dirs = np.vstack([q_t, -q_t] + ([cert.u, -cert.u] if cert.u.size else []))
        norms = np.linalg.norm(dirs, axis=1)
        dirs = dirs[norms > 0] / norms[norms > 0, None]       # empty groups have u = 0
        c, rad, n = key_block_stats(block)
        block = np.vstack([block, c + rad * dirs])       # boundary points, same ball
        c2, rad2, n2 = key_block_stats(block)
        ubb = block_upper_bound(cert, q_t, c2, rad2, n2)
        ub = upper_bound(cert, q_t, block)
        I = indexer_scores(q_t, w_t, block)
        assert np.all(ubb >= ub - 1e-9 * (1 + np.abs(ub)))
        assert np.all(ub >= I - 1e-9 * (1 + np.abs(I)))
        # and it is no looser than the center's bound plus the radius terms
        slack = rad2 * (cert.omega @ np.linalg.norm(q_t[cert.retained], axis=1)
                        if cert.retained.size else 0.0)
        slack += rad2 * float(np.sum(np.linalg.norm(cert.u, axis=1))) if cert.u.size else 0.0
        slack += cert.beta * (n2 - np.linalg.norm(c2))
        ubc = upper_bound(cert, q_t, c2[None, :])[0]
        assert ubb <= ubc + slack + 1e-9 * (1 + abs(ubc))


def test_block_bound_of_a_point_block_is_the_key_bound():
    """A block whose keys all coincide has radius 0 and max norm ||k||: its
    bound is the per-key bound of that key (closed form)."""
    from oracle import block_upper_bound, key_block_stats
    rng = np.random.default_rng(7)
    q_t, w_t, k = _instance(rng)
    cert = certificate_setup(q_t, w_t, key_mean(k), 4, 2)
    for s in (0, 5, 37):
        c, rad, n = key_block_stats(np.repeat(k[s:s + 1], 128, axis=0))
        assert rad == pytest.approx(0.0, abs=1e-12)
        assert block_upper_bound(cert, q_t, c, rad, n) == pytest.approx(
            upper_bound(cert, q_t, k[s:s + 1])[0], rel=1e-12, abs=1e-12)
