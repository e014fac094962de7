"""Full-size workloads in the launch configuration bench.py times: the
certified selection equals the dense selection on every row (a property that
holds at any size), and sampled rows match the fp64 oracle."""
import numpy as np
import pytest
import torch

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import WORKLOADS, codes_numpy, generate
from oracle import dequantize, indexer_scores
from parity import assert_topk_matches

pytestmark = pytest.mark.gpu


def _sample_rows(T, n=6):
    return sorted(set(np.linspace(0, T - 1, n).astype(int).tolist()) | {T - 1})


@pytest.mark.parametrize("name", ["causal_16k_bf16", "prefill_128k_fp8", "tight_64k_bf16_levels",
                                  "chunk_1m_fp8"])
def test_full_size_certified_equals_dense_and_sampled_oracle(cuda_lib, name):
    wl = WORKLOADS[name]
    x = generate(wl, device="cuda")
    idx = binding.Index(wl.dtype, max_K=wl.K)
    args = (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], x["seq_offsets"], wl.K)
    dense = idx.dense_topk(*args)
    cert, stats = idx.topk(*args, stats=True)
    torch.cuda.synchronize()
    assert torch.equal(cert, dense), "certified selection differs from the dense selection"
    assert stats["visible_pairs"] == wl.visible_pairs
    assert stats["exact_pairs"] + stats["rejected_pairs"] == wl.visible_pairs
    ks = None if x["k_scale"] is None else x["k_scale"].cpu().numpy()
    k = dequantize(codes_numpy(x["k"]), ks, wl.dtype)
    out = cert.cpu().numpy()
    for t in _sample_rows(wl.T):
        qs = None if x["q_scale"] is None else x["q_scale"][t:t + 1].cpu().numpy()
        q = dequantize(codes_numpy(x["q"][t:t + 1]), qs, wl.dtype)[0]
        w = x["w"][t].cpu().numpy().astype(np.float64)
        p = wl.q_pos0 + t
        assert_topk_matches(out[t], indexer_scores(q, w, k[: p + 1]), wl.K, t=t,
                            exact=wl.levels > 0)


def test_full_size_decode_equals_dense_and_oracle(cuda_lib):
    """The decode workload as bench.py times it: row 0 is the previous step,
    whose dense selection seeds the decode call on rows 1.."""
    wl = WORKLOADS["decode_1m_fp8"]
    x = generate(wl, device="cuda")
    idx = binding.Index(wl.dtype, max_K=wl.K)
    m = wl.T - 1

    def rows(lo, hi, pos0):
        sl = lambda v: None if v is None else v[lo:hi]
        return (sl(x["q"]), sl(x["q_scale"]), sl(x["w"]), x["k"], x["k_scale"],
                [[0, 0, pos0], [hi - lo, wl.S, 0]], wl.K)

    prev = idx.dense_topk(*rows(0, 1, wl.q_pos0))
    cur = rows(1, wl.T, wl.q_pos0 + 1)
    dense = idx.dense_topk(*cur)
    out, stats = idx.decode_topk(*cur, prev.expand(m, wl.K).contiguous(), stats=True)
    torch.cuda.synchronize()
    assert torch.equal(out, dense), "decode selection differs from the dense selection"
    assert stats["exact_pairs"] == sum(wl.q_pos0 + 2 + r for r in range(m))
    assert stats["candidates"] < 0.05 * stats["exact_pairs"], stats
    ks = x["k_scale"].cpu().numpy()
    k = dequantize(codes_numpy(x["k"]), ks, wl.dtype)
    o = out.cpu().numpy()
    for r in range(m):
        t = r + 1
        q = dequantize(codes_numpy(x["q"][t:t + 1]), x["q_scale"][t:t + 1].cpu().numpy(),
                       wl.dtype)[0]
        w = x["w"][t].cpu().numpy().astype(np.float64)
        p = wl.q_pos0 + t
        assert_topk_matches(o[r], indexer_scores(q, w, k[: p + 1]), wl.K, t=t)
