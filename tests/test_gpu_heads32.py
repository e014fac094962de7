"""GPU parity with a 32-head indexer (H = 32): the kernels read each query row
into 64 head slots whose upper half arrives as zeros and reduce only the 32
real heads.  Every path must match the fp64 oracle of the 32-head score, the
certified and decode selections must equal the dense one bit for bit, and the
certificate must match the oracle's on 32 heads."""
import numpy as np
import pytest
import torch

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import generate, small_case
from oracle import certificate_setup, key_mean
from parity import OracleView, assert_scores_close, assert_topk_matches, to_numpy

pytestmark = pytest.mark.gpu

CASES = [("causal_1k_bf16", 301, 1500, 64), ("prefill_128k_fp8_h32", 203, 2600, 300),
         ("tight_64k_bf16_levels", 157, 2100, 512)]


def _inputs(base, T, S, K, **kw):
    kw.setdefault("q_pos0", S - T)
    wl = small_case(base, T, S, K=K, H=32, **kw)
    x = generate(wl)
    assert x["q"].shape[1] == 32 and x["w"].shape[1] == 32
    xd = {k: (v.cuda() if torch.is_tensor(v) and k != "seq_offsets" else v) for k, v in x.items()}
    return wl, x, xd


def _args(x, K):
    return (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], x["seq_offsets"], K)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_h32_scores_match_oracle(cuda_lib, case):
    wl, x, xd = _inputs(*case)
    idx = binding.Index(wl.dtype, H=32)
    ov = OracleView(x, wl.dtype)
    S = wl.S
    for which in ("tc", "ref"):
        out = torch.full((wl.T, S), float("nan"), dtype=torch.float32, device="cuda")
        scratch = torch.zeros(256, dtype=torch.uint8, device="cuda")
        if which == "tc":
            idx.scores(xd["q"], xd["q_scale"], xd["w"], xd["k"], xd["k_scale"], 0, wl.T,
                       wl.q_pos0, S, out, S, scratch)
        else:
            idx.reference_scores(xd["q"], xd["q_scale"], xd["w"], xd["k"], xd["k_scale"], 0, wl.T,
                                 wl.q_pos0, S, out, S)
        got = to_numpy(out)
        for t in list(range(0, wl.T, 13)) + [wl.T - 1]:
            assert_scores_close(got[t], ov, t, exact=wl.levels > 0)


@pytest.mark.parametrize("screening", [2, 1, 0], ids=["adaptive", "always", "off"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_h32_certified_equals_dense_and_oracle(cuda_lib, case, screening):
    base, T, S, K = case
    wl, x, xd = _inputs(base, T, S, K)
    idx = binding.Index(wl.dtype, H=32, max_K=2048, screening=screening, short_dense_keys=0)
    dense = to_numpy(idx.dense_topk(*_args(xd, K)))
    cert, stats = idx.topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(cert), dense)
    ov = OracleView(x, wl.dtype)
    for t in range(0, wl.T, 5):
        assert_topk_matches(dense[t], ov.scores(t), K, mag=ov.magnitude(t), t=t, exact=wl.levels > 0)
    assert stats["exact_pairs"] + stats["rejected_pairs"] == wl.visible_pairs


def test_h32_host_staged_and_decode_equal_dense(cuda_lib):
    wl, x, xd = _inputs("prefill_128k_fp8_h32", 96, 3000, 256)
    K = 256
    idx = binding.Index(wl.dtype, H=32, max_K=2048)
    dense = to_numpy(idx.dense_topk(*_args(xd, K)))
    pin = {k: (v.contiguous().pin_memory() if torch.is_tensor(v) and k != "seq_offsets" else v)
           for k, v in x.items()}
    ws = torch.zeros(idx.host_workspace_size(wl.T, wl.S, wl.S, K, chunk_rows=32),
                     dtype=torch.uint8, device="cuda")
    out = idx.topk_host(*_args(pin, K), workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(out.numpy(), dense)
    # decode: rows 1.. seeded by row 0's selection
    prev = torch.as_tensor(dense[:1]).cuda().expand(wl.T - 1, K).contiguous()
    sub = {k: (v[1:] if torch.is_tensor(v) and k in ("q", "q_scale", "w") and v is not None else v)
           for k, v in xd.items()}
    sub["seq_offsets"] = [[0, 0, wl.q_pos0 + 1], [wl.T - 1, wl.S, 0]]
    dec = to_numpy(idx.decode_topk(*_args(sub, K), prev))
    assert np.array_equal(dec, dense[1:])


def test_h32_certificate_matches_oracle(cuda_lib):
    g = torch.Generator().manual_seed(7)
    T, S, H, d = 16, 900, 32, 128
    base = torch.randn((T, 1, d), generator=g)
    q = (base + 0.3 * torch.randn((T, H, d), generator=g)).to(torch.bfloat16)
    w = torch.randn((T, H), generator=g) / 8
    k = torch.randn((S, d), generator=g).to(torch.bfloat16)
    so = [[0, 0, S - T], [T, S, 0]]
    x = dict(q=q, q_scale=None, w=w, k=k, k_scale=None, seq_offsets=so,
             positions=torch.arange(S - T, S))
    idx = binding.Index("bf16", H=32)
    cert, ret = idx.certificate(q.cuda(), None, w.cuda(), k.cuda(), None, so)
    cert, ret = to_numpy(cert), to_numpy(ret)
    ov = OracleView(x, "bf16")
    kb = key_mean(ov.k)
    for t in range(T):
        c = certificate_setup(ov.q[t], ov.w[t], kb, 4, 2)
        assert ret[t][ret[t] >= 0].tolist() == c.retained.tolist()
        np.testing.assert_allclose(cert[t, 0:len(c.retained)], c.omega, rtol=2e-4, atol=1e-6)
        assert cert[t, 4] >= c.beta * (1 - 1e-5)
        assert cert[t, 10] == pytest.approx(c.beta_sum, rel=1e-3)
        assert cert[t, 12] + cert[t, 13] == sum(gr.size for gr in c.groups)
