"""Full-size workloads in the launch configuration bench.py times (inputs
drawn on the device, the default certified call): the certified selection
equals the dense selection on every row (a property that holds at any size),
and both match the fp64 oracle on every row of the 1K and 16K workloads and
on a fixed sample of the large ones: 512 evenly spaced rows, the last 8 rows,
and, for sequences that start at position 0, every 16th row below K (rows
with at most K visible keys, whose output is padded)."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch
from threadpoolctl import threadpool_limits

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import WORKLOADS, codes_numpy, generate
from oracle import dequantize, indexer_scores
from parity import assert_topk_matches, magnitude

pytestmark = pytest.mark.gpu

EVERY_ROW = {"causal_1k_bf16", "causal_16k_bf16"}


def oracle_rows(wl) -> list:
    if wl.name in EVERY_ROW:
        return list(range(wl.T))
    rows = set(np.linspace(0, wl.T - 1, 512).astype(int).tolist()) | set(range(wl.T - 8, wl.T))
    if wl.q_pos0 == 0:
        rows |= set(range(0, min(wl.K, wl.T), 16))
    return sorted(rows)


def check_against_oracle(x, wl, outs: dict, rows):
    """Every listed row of every output in `outs` against the oracle, rows
    spread over the host cores (one BLAS thread each)."""
    ks = None if x["k_scale"] is None else x["k_scale"].cpu().numpy()
    k = dequantize(codes_numpy(x["k"]), ks, wl.dtype)
    q_codes = codes_numpy(x["q"])
    qs = None if x["q_scale"] is None else x["q_scale"].cpu().numpy()
    w_all = x["w"].cpu().numpy().astype(np.float64)
    outs = {name: o.cpu().numpy() for name, o in outs.items()}

    def one(t):
        q = dequantize(q_codes[t:t + 1], None if qs is None else qs[t:t + 1], wl.dtype)[0]
        w = w_all[t]
        kv = k[: wl.q_pos0 + t + 1]
        scores = indexer_scores(q, w, kv)
        for name, o in outs.items():
            assert_topk_matches(o[t], scores, wl.K, t=(name, t), exact=wl.levels > 0,
                                mag=lambda: magnitude(q, w, kv))
        return t

    with threadpool_limits(1):
        with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
            done = list(ex.map(one, rows))
    assert done == list(rows)


@pytest.mark.parametrize("name", ["causal_1k_bf16", "causal_16k_bf16", "prefill_128k_fp8",
                                  "tight_64k_bf16_levels", "chunk_1m_fp8",
                                  "redundant_chunk128k_fp8", "redundant_128k_fp8"])
def test_full_size_certified_equals_dense_and_oracle(cuda_lib, name):
    wl = WORKLOADS[name]
    x = generate(wl, device="cuda")
    idx = binding.Index(wl.dtype, max_K=max(2048, wl.K))
    args = (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], x["seq_offsets"], wl.K)
    dense = idx.dense_topk(*args)
    cert, stats = idx.topk(*args, stats=True)
    torch.cuda.synchronize()
    assert torch.equal(cert, dense), "certified selection differs from the dense selection"
    if wl.S <= idx.cfg.short_dense_keys:
        # the default call took the dense path: run the certified machinery too
        machinery = binding.Index(wl.dtype, max_K=max(2048, wl.K), short_dense_keys=0)
        cert, stats = machinery.topk(*args, stats=True)
        assert torch.equal(cert, dense), "certified selection differs from the dense selection"
    assert stats["visible_pairs"] == wl.visible_pairs
    assert stats["exact_pairs"] + stats["rejected_pairs"] == wl.visible_pairs
    del x["sinks"]
    check_against_oracle(x, wl, {"certified": cert}, oracle_rows(wl))


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
        kv = k[: wl.q_pos0 + t + 1]
        assert_topk_matches(o[r], indexer_scores(q, w, kv), wl.K, t=t,
                            mag=lambda: magnitude(q, w, kv))
