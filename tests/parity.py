"""Helpers for GPU-vs-oracle parity tests: decode the generated inputs through
the oracle, compute oracle scores for chosen rows, and compare.

Tolerances (derived from the arithmetic, not tuned):
  scores   |gpu - oracle| <= 2^-15 * B(t,s),  B = sum_h |w_h| sum_i |q_hi k_i|
           (fp32 accumulation of <= 192 terms errs by <= 192 * 2^-24 * B ~ 2^-16.4 B;
           2^-15 leaves headroom for the tensor core's accumulation order).
  Top-K    the index sets have equal size and may differ only in keys whose
           oracle score lies within 1e-4 |v_K| of the K-th score v_K (the
           stated tolerance), widened by the rounding floor 2^-14 * B of the
           keys involved: a GPU score may sit 2^-15 B from the exact one, so
           two keys can swap order when their exact scores differ by less
           than the sum of their bounds.
  integer-level inputs: every score is exact in fp32, so equality is exact.
"""
from __future__ import annotations

import numpy as np
import torch

from exact_certified_top_b200.workloads import codes_numpy
from oracle import dequantize, indexer_scores, select_topk


class OracleView:
    """fp64 real-valued copies of generated inputs, for the oracle."""

    def __init__(self, x: dict, dtype: str):
        self.dtype = dtype
        qs = None if x["q_scale"] is None else x["q_scale"].cpu().numpy()
        ks = None if x["k_scale"] is None else x["k_scale"].cpu().numpy()
        self.q = dequantize(codes_numpy(x["q"]), qs, dtype)
        self.k = dequantize(codes_numpy(x["k"]), ks, dtype)
        self.w = x["w"].cpu().numpy().astype(np.float64)
        self.positions = x["positions"].cpu().numpy()

    def scores(self, t: int) -> np.ndarray:
        p = int(self.positions[t])
        return indexer_scores(self.q[t], self.w[t], self.k[: p + 1])

    def magnitude(self, t: int) -> np.ndarray:
        p = int(self.positions[t])
        return magnitude(self.q[t], self.w[t], self.k[: p + 1])


def assert_scores_close(gpu_row: np.ndarray, ov: OracleView, t: int, exact: bool = False):
    ref = ov.scores(t)
    got = gpu_row[: ref.shape[0]].astype(np.float64)
    if exact:
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, f"row {t}: {bad.size} inexact scores, first {bad[:5]}"
        return
    tol = 2.0 ** -15 * ov.magnitude(t) + 1e-30
    err = np.abs(got - ref)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (f"row {t}: {bad.size} scores out of tolerance, first key {bad[0]}: "
                           f"gpu {got[bad[0]]} oracle {ref[bad[0]]} tol {tol[bad[0]]}")


def magnitude(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray) -> np.ndarray:
    """B(t,s) = sum_h |w_h| sum_i |q_hi k_si| for every key: the bound of the
    fp32 rounding error of a score (see the module docstring)."""
    return np.abs(k) @ np.abs(q_t).T @ np.abs(w_t)


def kth_score(scores: np.ndarray, K: int) -> tuple[float, int]:
    """(v_K, the key holding it) of a row with more than K keys."""
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -scores))
    return float(scores[order[K - 1]]), int(order[K - 1])


def assert_topk_matches(gpu_idx: np.ndarray, scores: np.ndarray, K: int, t=None, exact=False,
                        mag=None):
    """gpu_idx: [K] int (ascending, -1 padded).  scores: oracle scores of the
    row; mag: magnitude() of the row's keys (or a callable returning it,
    evaluated only when the index sets differ).  The index sets may differ only
    in keys whose oracle score lies within 1e-4 |v_K| of the K-th score v_K,
    plus the fp32 rounding floor 2 * 2^-15 * B of the keys involved (both
    the differing keys and the key at v_K can be off by 2^-15 B each)."""
    n = scores.shape[0]
    want = select_topk(scores, K)
    got = np.asarray(gpu_idx, np.int64)
    assert np.all(np.diff(got[got >= 0]) > 0), f"row {t}: indices not strictly ascending"
    assert np.sum(got >= 0) == min(K, n), f"row {t}: wrong count"
    assert np.all(got[min(K, n):] == -1), f"row {t}: bad padding"
    if exact or n <= K:
        assert np.array_equal(got, want), f"row {t}: selection differs"
        return
    diff = np.setxor1d(got[got >= 0], want[want >= 0])
    if diff.size:
        assert mag is not None, "a non-exact comparison needs the magnitude bound"
        if callable(mag):
            mag = mag()
        vK, kk = kth_score(scores, K)
        band = 1e-4 * abs(vK) + 2.0 ** -14 * max(float(np.max(mag[diff])), float(mag[kk]))
        dev = np.abs(scores[diff] - vK)
        assert np.all(dev <= band), (f"row {t}: {diff.size} indices differ beyond the band: "
                                     f"max |s - vK| = {dev.max()} band {band}")


def to_numpy(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
