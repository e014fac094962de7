"""Helpers for GPU-vs-oracle parity tests: decode the generated inputs through
the oracle, compute oracle scores for chosen rows, and compare.

Tolerances (derived from the arithmetic, not tuned):
  scores   |gpu - oracle| <= 2^-15 * B(t,s),  B = sum_h |w_h| sum_i |q_hi k_i|
           (fp32 accumulation of <= 192 terms errs by <= 192 * 2^-24 * B ~ 2^-16.4 B;
           2^-15 leaves headroom for the tensor core's accumulation order).
  Top-K    the index sets have equal size and may differ only in keys whose
           oracle score lies within 1e-4 * max(|v_K|, 1e-3 * max_s |I(t,s)|) of
           the K-th score v_K.
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
        return np.abs(self.k[: p + 1]) @ np.abs(self.q[t]).T @ np.abs(self.w[t])


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


def topk_band(scores: np.ndarray, K: int) -> tuple[float, float]:
    """(v_K, band half-width) for the index-set comparison."""
    n = scores.shape[0]
    if n <= K:
        return -np.inf, 0.0
    vK = float(np.partition(scores, n - K)[n - K])
    return vK, 1e-4 * max(abs(vK), 1e-3 * float(np.max(np.abs(scores))))


def assert_topk_matches(gpu_idx: np.ndarray, scores: np.ndarray, K: int, t=None, exact=False):
    """gpu_idx: [K] int (ascending, -1 padded).  scores: oracle scores of the row."""
    n = scores.shape[0]
    want = select_topk(scores, K)
    got = np.asarray(gpu_idx, np.int64)
    assert np.all(np.diff(got[got >= 0]) > 0), f"row {t}: indices not strictly ascending"
    assert np.sum(got >= 0) == min(K, n), f"row {t}: wrong count"
    assert np.all(got[min(K, n):] == -1), f"row {t}: bad padding"
    if exact or n <= K:
        assert np.array_equal(got, want), f"row {t}: selection differs"
        return
    vK, band = topk_band(scores, K)
    diff = np.setxor1d(got[got >= 0], want[want >= 0])
    if diff.size:
        dev = np.abs(scores[diff] - vK)
        assert np.all(dev <= band), (f"row {t}: {diff.size} indices differ beyond the band: "
                                     f"max |s - vK| = {dev.max()} band {band}")


def to_numpy(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
