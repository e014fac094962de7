"""GPU parity of the decode-step indexer (dosa_index_decode_topk): a few
query rows against a long key cache, seeded by the previous step's
selection.  The selection must equal the dense path's bit for bit and the
oracle's up to the tolerance, whatever the seeds are (good, exact, poor,
duplicated, padded)."""
import numpy as np
import pytest
import torch

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import generate, small_case
from parity import OracleView, assert_topk_matches, to_numpy

pytestmark = pytest.mark.gpu


def _decode_case(base, S, m, K, seed=0, noise=0.3):
    """m + 1 rows at the end of S keys: row 0 is the previous step, rows 1..m
    are perturbations of it (consecutive decode queries)."""
    wl = small_case(base, m + 1, S, K=K, q_pos0=S - m - 1, seed=seed, decode_noise=noise)
    x = generate(wl)
    xd = {k: (v.cuda() if torch.is_tensor(v) and k != "seq_offsets" else v) for k, v in x.items()}
    return wl, x, xd


def _rows(xd, lo, hi, S, pos0):
    sub = {k: (v[lo:hi] if torch.is_tensor(v) and k in ("q", "q_scale", "w") and v is not None
               else v) for k, v in xd.items()}
    sub["seq_offsets"] = [[0, 0, pos0], [hi - lo, S, 0]]
    return sub


def _args(x, K):
    return (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], x["seq_offsets"], K)


@pytest.mark.parametrize("case", [("prefill_128k_fp8", 20000, 4, 2048),
                                  ("causal_1k_bf16", 9000, 3, 256),
                                  ("prefill_128k_fp8", 70000, 1, 512)],
                         ids=lambda c: f"{c[0]}-S{c[1]}-m{c[2]}-K{c[3]}")
def test_decode_seeded_by_previous_step_equals_dense(cuda_lib, case):
    base, S, m, K = case
    wl, x, xd = _decode_case(base, S, m, K)
    idx = binding.Index(wl.dtype, max_K=2048)
    prev = _rows(xd, 0, 1, S, S - m - 1)
    cur = _rows(xd, 1, m + 1, S, S - m)
    prev_sel = idx.dense_topk(*_args(prev, K))
    seeds = prev_sel.expand(m, K).contiguous()
    dense = to_numpy(idx.dense_topk(*_args(cur, K)))
    out, stats = idx.decode_topk(*_args(cur, K), seeds, stats=True)
    out = to_numpy(out)
    assert np.array_equal(out, dense)
    ov = OracleView(x, wl.dtype)
    for r in range(m):
        assert_topk_matches(out[r], ov.scores(r + 1), K, t=r + 1, exact=False,
                            mag=ov.magnitude(r + 1))
    assert stats["exact_pairs"] == sum(S - m + r + 1 for r in range(m))
    # the candidates are the keys at or above the seed threshold: at least K
    # per row, and no more than the keys the oracle puts above the lowest
    # possible GPU threshold (seed score - evaluation error - seed margin)
    sel = to_numpy(prev_sel)[0]
    upper = 0
    for r in range(m):
        t = r + 1
        ref, mag = ov.scores(t), ov.magnitude(t)
        err = 2.0 ** -15 * mag
        qn = np.linalg.norm(ov.q[t], axis=1)
        kn = np.linalg.norm(ov.k[sel], axis=1)
        margin = 2.0 ** -13 * float(np.abs(ov.w[t]) @ qn) * kn * (1 + 2.0 ** -10)
        low = float(np.min(ref[sel] - err[sel] - margin))
        upper += int(np.count_nonzero(ref + err >= low))
    assert m * K <= stats["candidates"] <= upper, (stats, upper)
    if K * 64 <= S:
        # a correlated previous step leaves a small fraction for selection
        assert stats["candidates"] < 0.25 * stats["exact_pairs"], stats


def test_decode_with_unrelated_seeds_stays_exact(cuda_lib):
    """Queries drawn independently of the previous step: the seeds bound
    little (nearly every key is a candidate, or the rows are repaired), and
    the selection is still the dense one."""
    S, m, K = 30000, 4, 1024
    wl, x, xd = _decode_case("prefill_128k_fp8", S, m, K, seed=7, noise=0.0)
    idx = binding.Index(wl.dtype, max_K=2048)
    prev = _rows(xd, 0, 1, S, S - m - 1)
    cur = _rows(xd, 1, m + 1, S, S - m)
    seeds = idx.dense_topk(*_args(prev, K)).expand(m, K).contiguous()
    out = idx.decode_topk(*_args(cur, K), seeds)
    assert torch.equal(out, idx.dense_topk(*_args(cur, K)))


@pytest.mark.parametrize("kind", ["exact", "duplicates", "padded", "invisible"])
def test_decode_seed_edge_cases(cuda_lib, kind):
    """Seeds that are the answer itself (tightest bound), that repeat an index
    or are short (no bound: every row is repaired densely), or point past the
    row's position: the result is the dense selection every time."""
    S, m, K = 6000, 4, 300
    wl, x, xd = _decode_case("prefill_128k_fp8", S, m, K, seed=3)
    idx = binding.Index(wl.dtype, max_K=2048)
    cur = _rows(xd, 1, m + 1, S, S - m)
    dense = idx.dense_topk(*_args(cur, K))
    if kind == "exact":
        seeds = dense.clone()
    elif kind == "duplicates":
        seeds = dense.clone()
        seeds[:, 1] = seeds[:, 0]
    elif kind == "padded":
        seeds = dense.clone()
        seeds[:, K // 2:] = -1
    else:
        seeds = dense.clone()
        seeds[:, 0] = S + 5
    out = idx.decode_topk(*_args(cur, K), seeds)
    assert torch.equal(out, dense)


def test_decode_short_rows_and_varlen_batch(cuda_lib):
    """Two sequences in one call, one with fewer visible keys than K."""
    K = 128
    a = small_case("causal_1k_bf16", 3, 3000, K=K, q_pos0=2997, seed=5)
    b = small_case("causal_1k_bf16", 2, 100, K=K, q_pos0=98, seed=6)
    xa, xb = generate(a), generate(b)
    q = torch.cat([xa["q"], xb["q"]]).cuda()
    w = torch.cat([xa["w"], xb["w"]]).cuda()
    k = torch.cat([xa["k"], xb["k"]]).cuda()
    so = [[0, 0, 2997], [3, 3000, 98], [5, 3100, 0]]
    idx = binding.Index("bf16")
    dense = idx.dense_topk(q, None, w, k, None, so, K)
    out = idx.decode_topk(q, None, w, k, None, so, K, dense)
    assert torch.equal(out, dense)
    o = to_numpy(out)
    for r, vis in ((3, 99), (4, 100)):        # fewer visible keys than K: padded with -1
        assert (o[r, vis:] == -1).all() and (o[r, :vis] >= 0).all()
