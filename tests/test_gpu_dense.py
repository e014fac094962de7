"""GPU parity of the dense path: tensor-core scorer, CUDA-core reference scorer,
radix Top-K and dense_topk, against the fp64 oracle on the same seeded inputs.
Sizes span several key tiles, several query tiles and ragged tails."""
import numpy as np
import pytest
import torch

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import generate, small_case
from oracle import select_topk
from parity import OracleView, assert_scores_close, assert_topk_matches, to_numpy

pytestmark = pytest.mark.gpu

CASES = [
    # (base workload, T, S): ragged against both the 8-query and 128-key tiles
    ("causal_1k_bf16", 1003, 1003),
    ("prefill_128k_fp8", 777, 777),
    ("tight_64k_bf16_levels", 517, 517),
    ("chunk_1m_fp8", 203, 1500),     # chunked prefill: rows at positions 1297..1499
]


def _inputs(base, T, S, device="cuda"):
    wl = small_case(base, T, S, K=64)
    x = generate(wl, device="cpu")
    xd = {k: (v.to(device) if torch.is_tensor(v) and k != "seq_offsets" else v)
          for k, v in x.items()}
    return wl, xd, OracleView(x, wl.dtype)


def _scores(idx, wl, x, which):
    S = wl.S
    out = torch.full((wl.T, S), float("nan"), dtype=torch.float32, device="cuda")
    scratch = torch.zeros(256, dtype=torch.uint8, device="cuda")
    fn = idx.scores if which == "tc" else idx.reference_scores
    args = (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], 0, wl.T, wl.q_pos0, S, out, S)
    fn(*args, scratch) if which == "tc" else fn(*args)
    torch.cuda.synchronize()
    if which == "tc":
        binding.check_device(scratch)
    return to_numpy(out)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("which", ["tc", "ref"])
def test_scores_match_oracle(cuda_lib, case, which):
    wl, x, ov = _inputs(*case)
    idx = binding.Index(wl.dtype)
    got = _scores(idx, wl, x, which)
    exact = wl.levels > 0
    rows = list(range(0, wl.T, max(1, wl.T // 97))) + [wl.T - 1]
    for t in rows:
        assert_scores_close(got[t], ov, t, exact=exact)
        p = wl.q_pos0 + t
        assert np.all(np.isnan(got[t, p + 1:])), "scores written past the causal limit"


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_tensor_core_scorer_matches_reference_scorer(cuda_lib, case):
    wl, x, ov = _inputs(*case)
    idx = binding.Index(wl.dtype)
    a = _scores(idx, wl, x, "tc")
    b = _scores(idx, wl, x, "ref")
    for t in range(0, wl.T, 7):
        p = wl.q_pos0 + t
        tol = 2.0 ** -14 * ov.magnitude(t)
        assert np.all(np.abs(a[t, : p + 1] - b[t, : p + 1]) <= tol)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("K", [1, 64, 300])
def test_dense_topk_matches_oracle(cuda_lib, case, K):
    wl, x, ov = _inputs(*case)
    idx = binding.Index(wl.dtype, max_K=2048)
    out = to_numpy(idx.dense_topk(x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"],
                                  x["seq_offsets"], K))
    for t in range(wl.T):
        assert_topk_matches(out[t], ov.scores(t), K, mag=ov.magnitude(t), t=t, exact=wl.levels > 0)


def test_dense_topk_small_workspace_many_chunks(cuda_lib):
    wl, x, ov = _inputs("causal_1k_bf16", 301, 301)
    idx = binding.Index("bf16")
    ws = torch.zeros(idx.workspace_size(wl.T, wl.S, 32, False, chunk_rows=16), dtype=torch.uint8,
                     device="cuda")
    out = to_numpy(idx.dense_topk(x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"],
                                  x["seq_offsets"], 32, workspace=ws))
    binding.check_device(ws)
    for t in range(wl.T):
        assert_topk_matches(out[t], ov.scores(t), 32, mag=ov.magnitude(t), t=t)


def test_dense_topk_varlen_batch(cuda_lib):
    """Three sequences packed in one call, each with its own keys and offsets."""
    parts = [small_case("causal_1k_bf16", 130, 130, seed=1),
             small_case("causal_1k_bf16", 40, 300, seed=2, q_pos0=260),
             small_case("causal_1k_bf16", 9, 9, seed=3)]
    xs = [generate(wl) for wl in parts]
    q = torch.cat([x["q"] for x in xs]).cuda()
    w = torch.cat([x["w"] for x in xs]).cuda()
    k = torch.cat([x["k"] for x in xs]).cuda()
    so, qr, kr = [], 0, 0
    for wl in parts:
        so.append([qr, kr, wl.q_pos0])
        qr += wl.T
        kr += wl.S
    so.append([qr, kr, 0])
    idx = binding.Index("bf16")
    out = to_numpy(idx.dense_topk(q, None, w, k, None, so, 50))
    r = 0
    for wl, x in zip(parts, xs):
        ov = OracleView(x, "bf16")
        for t in range(wl.T):
            assert_topk_matches(out[r + t], ov.scores(t), 50, mag=ov.magnitude(t), t=(wl.name, t))
        r += wl.T


def test_topk_rows_ties_zero_and_short_rows(cuda_lib):
    rng = np.random.default_rng(0)
    rows, L = 9, 5000
    s = rng.integers(-20, 20, size=(rows, L)).astype(np.float32) * 0.25   # many exact ties
    s[1] = 0.0
    s[1, ::2] = -0.0                                                     # -0 ties +0
    s[2, :] = rng.standard_normal(L).astype(np.float32)
    lens = np.array([L, L, L, 10, 1, 4096, 4097, 2000, 300], np.int64)
    dev = torch.from_numpy(s).cuda()
    for K in (1, 7, 2048, 4096):
        out = to_numpy(binding.topk_rows(dev, torch.from_numpy(lens).cuda(), K))
        for i in range(rows):
            want = select_topk(s[i, : lens[i]].astype(np.float64), K)
            assert np.array_equal(out[i], want), (K, i)
