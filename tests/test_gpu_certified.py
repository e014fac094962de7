"""GPU parity of the certified path (dosa_index_topk): identical selection to
the GPU's dense path, agreement with the fp64 oracle, certificate quantities
against the oracle's, the prune-rate invariant, and the overflow repair."""
import numpy as np
import pytest
import torch

from exact_certified_top_b200 import binding
from exact_certified_top_b200.workloads import codes_numpy, generate, small_case
from oracle import (certificate_setup, certified_topk_row, dequantize, indexer_scores, key_mean,
                    select_topk)
from parity import OracleView, assert_topk_matches, to_numpy

pytestmark = pytest.mark.gpu

CASES = [
    ("causal_1k_bf16", 1003, 1003, 64),
    ("prefill_128k_fp8", 777, 3000, 300),
    ("tight_64k_bf16_levels", 517, 2600, 2048),
    ("chunk_1m_fp8", 203, 5000, 2048),
]


def _inputs(base, T, S, K, **kw):
    kw.setdefault("q_pos0", S - T)          # rows at the tail: the longest contexts
    wl = small_case(base, T, S, K=K, **kw)
    x = generate(wl)
    xd = {k: (v.cuda() if torch.is_tensor(v) and k != "seq_offsets" else v) for k, v in x.items()}
    return wl, x, xd


def _args(x, K):
    return (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], x["seq_offsets"], K)


def Index(*a, **kw):
    """A handle that runs the certified machinery at every size: these tests
    look inside it on small shapes, which the adaptive mode would otherwise
    hand to the dense path (short_dense_keys)."""
    kw.setdefault("short_dense_keys", 0)
    return binding.Index(*a, **kw)


MODES = dict(argvalues=[3, 2, 1, 0], ids=["ranked", "adaptive", "streaming", "off"])


@pytest.mark.parametrize("screening", **MODES)
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_certified_equals_dense_and_oracle(cuda_lib, case, screening):
    base, T, S, K = case
    wl, x, xd = _inputs(base, T, S, K)
    idx = Index(wl.dtype, max_K=2048, screening=screening)
    dense = to_numpy(idx.dense_topk(*_args(xd, K)))
    cert, stats = idx.topk(*_args(xd, K), stats=True)
    cert = to_numpy(cert)
    assert np.array_equal(cert, dense), "certified selection differs from the dense selection"
    ov = OracleView(x, wl.dtype)
    for t in range(0, wl.T, max(1, wl.T // 120)):
        assert_topk_matches(cert[t], ov.scores(t), K, mag=ov.magnitude(t), t=t, exact=wl.levels > 0)
    assert stats["visible_pairs"] == wl.visible_pairs
    assert 0 <= stats["rejected_pairs"] <= stats["screened_pairs"]
    assert stats["exact_pairs"] + stats["rejected_pairs"] == wl.visible_pairs
    assert 0 <= stats["filtered_pairs"] <= stats["exact_pairs"]
    if screening == 0:
        assert stats["screened_pairs"] == 0
        assert stats["filtered_pairs"] == wl.visible_pairs
    if screening == 1:
        assert stats["filtered_pairs"] == 0
    if screening >= 2:
        assert stats["rescreened_pairs"] <= stats["exact_pairs"]


def test_certified_small_workspace_many_chunks(cuda_lib):
    wl, x, xd = _inputs("causal_1k_bf16", 301, 2500, 100, q_pos0=2199)
    idx = Index("bf16")
    ws = torch.zeros(idx.workspace_size(wl.T, wl.S, 100, True, chunk_rows=16), dtype=torch.uint8,
                     device="cuda")
    cert = to_numpy(idx.topk(*_args(xd, 100), workspace=ws))
    binding.check_device(ws)
    dense = to_numpy(idx.dense_topk(*_args(xd, 100)))
    assert np.array_equal(cert, dense)


def test_certified_varlen_batch(cuda_lib):
    parts = [small_case("causal_1k_bf16", 130, 2300, seed=1, q_pos0=2170),
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
    idx = Index("bf16")
    cert = to_numpy(idx.topk(q, None, w, k, None, so, 70))
    dense = to_numpy(idx.dense_topk(q, None, w, k, None, so, 70))
    assert np.array_equal(cert, dense)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_varlen_batch_with_empty_sequences(cuda_lib, dtype):
    """A packed batch whose first and middle sequences have keys but no query
    rows: the certified, host-staged and dense calls skip them, and every
    other row's selection is the oracle's (indices relative to its own
    sequence's first key)."""
    base = "causal_1k_bf16" if dtype == "bf16" else "prefill_128k_fp8"
    parts = [small_case(base, 0, 77, seed=4, q_pos0=77),
             small_case(base, 130, 2300, seed=1, q_pos0=2170),
             small_case(base, 0, 300, seed=5, q_pos0=300),
             small_case(base, 24, 500, seed=2, q_pos0=476)]
    xs = [generate(wl) for wl in parts]
    cat = lambda key: torch.cat([x[key] for x in xs])
    q, w, k = cat("q"), cat("w"), cat("k")
    qs = cat("q_scale") if dtype == "fp8" else None
    ks = cat("k_scale") if dtype == "fp8" else None
    so, qr, kr = [], 0, 0
    for wl in parts:
        so.append([qr, kr, wl.q_pos0])
        qr += wl.T
        kr += wl.S
    so.append([qr, kr, 0])
    K = 64
    dev = lambda t: None if t is None else t.cuda()
    idx = Index(dtype)
    cert = to_numpy(idx.topk(dev(q), dev(qs), dev(w), dev(k), dev(ks), so, K))
    dense = to_numpy(idx.dense_topk(dev(q), dev(qs), dev(w), dev(k), dev(ks), so, K))
    assert cert.shape == (qr, K)
    assert np.array_equal(cert, dense)
    pin = lambda t: None if t is None else t.contiguous().pin_memory()
    ws = torch.zeros(idx.host_workspace_size(qr, kr, 2300, K), dtype=torch.uint8, device="cuda")
    host = idx.topk_host(pin(q), pin(qs), pin(w), pin(k), pin(ks), so, K, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(host.numpy(), cert)
    r = 0
    for wl, x in zip(parts, xs):
        if wl.T:
            ov = OracleView(x, dtype)
            for t in range(0, wl.T, 5):
                assert_topk_matches(cert[r + t], ov.scores(t), K, mag=ov.magnitude(t), t=(wl.name, t))
        r += wl.T


def _redundant_heads_case(T=96, S=6000, seed=0, fp8=False):
    """Heads of a query are near copies of one direction and weights mostly
    positive: the certificate is tight and most keys are rejected."""
    g = torch.Generator().manual_seed(seed)
    d, H = 128, 64
    base = torch.randn((T, 1, d), generator=g)
    q = base + 0.02 * torch.randn((T, H, d), generator=g)
    w = torch.rand((T, H), generator=g) / 8
    w[:, ::16] *= -0.2
    k = torch.randn((S, d), generator=g)
    pos0 = S - T
    so = [[0, 0, pos0], [T, S, 0]]
    if fp8:
        from exact_certified_top_b200.workloads import _e4m3_per_token
        q8, qs = _e4m3_per_token(q)
        k8, ks = _e4m3_per_token(k)
        return dict(q=q8, q_scale=qs, w=w, k=k8, k_scale=ks, seq_offsets=so,
                    positions=torch.arange(pos0, S)), "fp8"
    return dict(q=q.to(torch.bfloat16), q_scale=None, w=w, k=k.to(torch.bfloat16), k_scale=None,
                seq_offsets=so, positions=torch.arange(pos0, S)), "bf16"


@pytest.mark.parametrize("screening", [3, 2, 1], ids=["ranked", "adaptive", "streaming"])
@pytest.mark.parametrize("fp8", [False, True])
def test_certified_prunes_and_stays_exact_when_heads_are_redundant(cuda_lib, fp8, screening):
    x, dtype = _redundant_heads_case(fp8=fp8)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    K = 64
    idx = Index(dtype, screening=screening)
    cert, stats = idx.topk(*_args(xd, K), stats=True)
    dense = idx.dense_topk(*_args(xd, K))
    assert torch.equal(cert, dense)
    prune = stats["rejected_pairs"] / stats["visible_pairs"]
    assert prune > 0.5, stats
    # the schedule's threshold is <= the true K-th and the GPU bound is >= the
    # oracle's, so the GPU rejects no more than the oracle's ideal screening
    ov = OracleView(x, dtype)
    kb = key_mean(ov.k)
    ideal = 0
    for t in range(0, x["q"].shape[0]):
        p = int(ov.positions[t])
        res = certified_topk_row(ov.q[t], ov.w[t], ov.k[: p + 1], K, k_bar=kb, r=4, G=2,
                                 margin_log2=-12)
        ideal += res["ideal_rejected"]
        assert np.array_equal(res["idx"], to_numpy(cert[t]).astype(np.int64))
    assert stats["rejected_pairs"] <= ideal * 1.002 + 16, (stats, ideal)


def test_certificate_matches_oracle(cuda_lib):
    for fp8 in (False, True):
        x, dtype = _redundant_heads_case(T=24, S=700, seed=3, fp8=fp8)
        # make heads less redundant so the residual bounds are non-trivial
        xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
        idx = Index(dtype)
        cert, ret = idx.certificate(xd["q"], xd["q_scale"], xd["w"], xd["k"], xd["k_scale"],
                                    x["seq_offsets"])
        cert, ret = to_numpy(cert), to_numpy(ret)
        ov = OracleView(x, dtype)
        kb = key_mean(ov.k)
        for t in range(x["q"].shape[0]):
            sq = 1.0 if x["q_scale"] is None else float(x["q_scale"][t])
            c = certificate_setup(ov.q[t], ov.w[t], kb, 4, 2)
            assert ret[t][ret[t] >= 0].tolist() == c.retained.tolist()
            np.testing.assert_allclose(cert[t, 0:len(c.retained)], c.omega, rtol=2e-4, atol=1e-6)
            # GPU beta (code domain) scaled to the real domain is an upper bound
            # of the oracle's residual bound, and not far above it
            assert cert[t, 4] * sq >= c.beta * (1 - 1e-5)
            assert cert[t, 10] * sq == pytest.approx(c.beta_sum, rel=1e-3)
            assert cert[t, 11] * sq >= c.beta_joint * (1 - 1e-5)
            assert cert[t, 12] + cert[t, 13] == sum(g.size for g in c.groups)


@pytest.mark.parametrize("fp8", [False, True])
def test_certified_mixed_items_hand_over_and_continue(cuda_lib, fp8):
    """Work items of 8 queries alternate between redundant heads (screening
    rejects most keys: the probe lets screening continue) and independent
    random heads (screening rejects almost nothing: the probe hands the item to
    the filter scorer).  Both finishers run in one call; the selection stays
    identical to the dense path and to the oracle.  Every item is probed
    (probe_sample = 0); with the sampled probe the selection is the same."""
    x, dtype = _redundant_heads_case(T=160, S=7000, seed=11, fp8=fp8)
    g = torch.Generator().manual_seed(12)
    rand_rows = torch.cat([torch.arange(i, i + 8) for i in range(8, 160, 16)])
    if fp8:
        from exact_certified_top_b200.workloads import _e4m3_per_token
        q8, qs = _e4m3_per_token(torch.randn((len(rand_rows), 64, 128), generator=g))
        x["q"][rand_rows] = q8
        x["q_scale"][rand_rows] = qs
    else:
        x["q"][rand_rows] = torch.randn((len(rand_rows), 64, 128), generator=g).to(torch.bfloat16)
    x["w"][rand_rows] = torch.randn((len(rand_rows), 64), generator=g) / 8
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    K = 128
    idx = Index(dtype, screening=2, probe_sample=0)
    cert, stats = idx.topk(*_args(xd, K), stats=True)
    dense = idx.dense_topk(*_args(xd, K))
    assert torch.equal(cert, dense)
    sampled, st_s = Index(dtype, screening=2).topk(*_args(xd, K), stats=True)
    assert torch.equal(sampled, dense)
    assert st_s["exact_pairs"] + st_s["rejected_pairs"] == st_s["visible_pairs"]
    assert stats["exact_pairs"] + stats["rejected_pairs"] == stats["visible_pairs"]
    # about half the rows prune most of their keys, the other half hardly any
    prune = stats["rejected_pairs"] / stats["visible_pairs"]
    assert 0.2 < prune < 0.6, stats
    # the filtered half is not screened past its probe tiles
    assert stats["screened_pairs"] < 0.75 * stats["visible_pairs"], stats
    ov = OracleView(x, dtype)
    cert = to_numpy(cert)
    for t in range(0, 160, 7):
        assert_topk_matches(cert[t], ov.scores(t), K, mag=ov.magnitude(t), t=t, exact=False)


@pytest.mark.parametrize("screening", **MODES)
@pytest.mark.parametrize("S", [5200, 70000])
def test_repair_pass_when_candidates_overflow(cuda_lib, screening, S):
    """All keys identical: every score ties, every key becomes a candidate and
    the candidate list overflows; the rows are rescored densely and the
    selection (ties to the smaller index) is still exact.  With 70,000 keys
    each repaired row's key tiles are split over several work items."""
    T, K = 40, 64
    g = torch.Generator().manual_seed(5)
    q = torch.randn((T, 64, 128), generator=g).to(torch.bfloat16)
    w = torch.randn((T, 64), generator=g) / 8
    k = torch.randn((1, 128), generator=g).expand(S, 128).contiguous().to(torch.bfloat16)
    so = [[0, 0, S - T], [T, S, 0]]
    idx = Index("bf16", screening=screening)
    qd, wd, kd = q.cuda(), w.cuda(), k.cuda()
    cert, stats = idx.topk(qd, None, wd, kd, None, so, K, stats=True)
    cert = to_numpy(cert)
    dense = to_numpy(idx.dense_topk(qd, None, wd, kd, None, so, K))
    assert np.array_equal(cert, dense)
    assert np.array_equal(cert, np.tile(np.arange(K, dtype=np.int32), (T, 1)))
    assert stats["repaired_rows"] == T


@pytest.mark.parametrize("case", [("prefill_128k_fp8", 203, 2600, 300), ("causal_1k_bf16", 300, 1900, 64)],
                         ids=lambda c: c[0])
def test_host_staged_call_equals_device_call(cuda_lib, case):
    """dosa_index_topk_host: inputs and output in pinned host memory, query
    rows streamed through two staging slots (a small workspace forces many
    chunks, so both slots are reused); same indices as the device call."""
    base, T, S, K = case
    wl, x, xd = _inputs(base, T, S, K)
    idx = Index(wl.dtype, max_K=2048)
    dev = to_numpy(idx.topk(*_args(xd, K)))
    pin = {k: (v.contiguous().pin_memory() if torch.is_tensor(v) and k != "seq_offsets" else v)
           for k, v in x.items()}
    so = x["seq_offsets"]
    ws = torch.zeros(idx.host_workspace_size(wl.T, wl.S, wl.S, K, chunk_rows=48),
                     dtype=torch.uint8, device="cuda")
    out, stats = idx.topk_host(*_args(pin, K), workspace=ws, stats=True)
    assert out.device.type == "cpu"
    assert np.array_equal(out.numpy(), dev)
    assert stats["exact_pairs"] + stats["rejected_pairs"] == wl.visible_pairs
    # again on the same workspace and stream (slots reused across calls)
    out2 = idx.topk_host(*_args(pin, K), workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(out2.numpy(), dev)


@pytest.mark.parametrize("screening", **MODES)
@pytest.mark.parametrize("case", [("prefill_128k_fp8", 203, 2600, 300),
                                  ("tight_64k_bf16_levels", 157, 2100, 512)],
                         ids=lambda c: c[0])
def test_dense_writeback_ablation_equals_dense(cuda_lib, case, screening):
    """sparse_writeback = 0: every exact score also goes to a dense chunk
    matrix (rejected pairs -inf) and the selection is its dense Top-K.  The
    indices must equal the sparse path's and the dense path's."""
    base, T, S, K = case
    wl, x, xd = _inputs(base, T, S, K)
    dense = to_numpy(Index(wl.dtype, max_K=2048).dense_topk(*_args(xd, K)))
    idx = Index(wl.dtype, max_K=2048, screening=screening, sparse_writeback=0)
    out, stats = idx.topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(out), dense)
    assert stats["exact_pairs"] + stats["rejected_pairs"] == wl.visible_pairs
    # a workspace for few rows: many chunks, each with its own dense matrix
    ws = torch.zeros(idx.workspace_size(24, wl.S, K, True), dtype=torch.uint8, device="cuda")
    out2 = idx.topk(*_args(xd, K), workspace=ws)
    assert np.array_equal(to_numpy(out2), dense)


def _clustered_blocks_case(T=48, n_tiles=50, seed=5, fp8=False):
    """Keys in 128-key tiles that are tight balls: 'hot' tiles point along the
    queries' common direction, 'cold' ones against it.  Query heads are near
    copies (a tight certificate) with mostly positive weights, so every cold
    tile's block bound is far below the threshold the hot keys set."""
    g = torch.Generator().manual_seed(seed)
    d, H = 128, 64
    base = torch.randn(d, generator=g)
    base = base / base.norm()
    qdir = base + 0.2 * torch.randn((T, 1, d), generator=g)
    q = 4.0 * qdir + 0.02 * torch.randn((T, H, d), generator=g)
    w = torch.rand((T, H), generator=g) / 8
    w[:, ::16] *= -0.2
    S = n_tiles * 128
    hot = torch.zeros(n_tiles, dtype=torch.bool)
    hot[0] = True
    hot[-6:] = True              # the diagonal tiles (seeds, warm-up)
    hot[::3] = True
    sign = torch.where(hot, 1.0, -1.0).repeat_interleave(128)[:, None]
    k = sign * (2.0 * base + 0.05 * torch.randn((S, d), generator=g))
    k = k + 0.3 * torch.randn((n_tiles, 1, d), generator=g).repeat_interleave(128, 0).view(S, d) * 0.1
    pos0 = S - T
    so = [[0, 0, pos0], [T, S, 0]]
    if fp8:
        from exact_certified_top_b200.workloads import _e4m3_per_token
        q8, qs = _e4m3_per_token(q)
        k8, ks = _e4m3_per_token(k)
        return dict(q=q8, q_scale=qs, w=w, k=k8, k_scale=ks, seq_offsets=so,
                    positions=torch.arange(pos0, S)), "fp8"
    return dict(q=q.to(torch.bfloat16), q_scale=None, w=w, k=k.to(torch.bfloat16), k_scale=None,
                seq_offsets=so, positions=torch.arange(pos0, S)), "bf16"


@pytest.mark.parametrize("screening", [1])
@pytest.mark.parametrize("fp8", [False, True])
def test_key_block_certificate_skips_tiles_and_stays_exact(cuda_lib, fp8, screening):
    """The key-block certificate acts in the streaming schedule (screening =
    1): whole tiles whose block bound rules them out are skipped."""
    x, dtype = _clustered_blocks_case(fp8=fp8)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    K = 64
    dense = to_numpy(Index(dtype).dense_topk(*_args(xd, K)))
    on = Index(dtype, screening=screening, block_bound=1)
    off = Index(dtype, screening=screening, block_bound=0)
    a, sa = on.topk(*_args(xd, K), stats=True)
    b, sb = off.topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(a), dense) and np.array_equal(to_numpy(b), dense)
    T, S = x["q"].shape[0], x["k"].shape[0]
    visible = sum(S - T + t + 1 for t in range(T))
    for st in (sa, sb):
        assert st["exact_pairs"] + st["rejected_pairs"] == visible
    assert sb["block_skipped_pairs"] == 0
    assert sa["block_skipped_pairs"] > 0, sa
    assert sa["block_skipped_pairs"] <= sa["rejected_pairs"]
    ov = OracleView(x, dtype)
    for t in range(0, T, 5):
        assert_topk_matches(to_numpy(a)[t], ov.scores(t), K, mag=ov.magnitude(t), t=t)


def test_key_block_bounds_agree_with_oracle(cuda_lib):
    """Every tile the GPU skipped has, in the fp64 oracle, a block bound below
    the query's true K-th score for every query of the item that sees it (so
    no Top-K key can have been skipped); checked through the selection and the
    counters on the clustered case with one work item."""
    from oracle import block_upper_bound, key_block_stats
    x, dtype = _clustered_blocks_case(T=8, seed=9)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    K = 64
    idx = Index(dtype, screening=1, block_bound=1)
    out, st = idx.topk(*_args(xd, K), stats=True)
    ov = OracleView(x, dtype)
    kb = key_mean(ov.k)
    S = ov.k.shape[0]
    n_tiles = S // 128
    # tiles whose oracle block bound is below v_K for all 8 queries
    droppable = 0
    for j in range(1, n_tiles):
        ok = True
        for t in range(8):
            p = int(ov.positions[t])
            lo = j * 128
            if lo > p:
                continue
            c = certificate_setup(ov.q[t], ov.w[t], kb, 4, 2)
            cen, rad, nmax = key_block_stats(ov.k[lo:lo + 128])
            vk = np.sort(ov.scores(t))[-K]
            if not block_upper_bound(c, ov.q[t], cen, rad, nmax) < vk:
                ok = False
                break
        droppable += ok
    assert droppable > 0
    # the GPU's skipped pairs never exceed what the ideal bound could drop
    assert st["block_skipped_pairs"] <= droppable * 128 * 8
    for t in range(8):
        assert_topk_matches(to_numpy(out)[t], ov.scores(t), K, mag=ov.magnitude(t), t=t)


@pytest.mark.parametrize("fp8", [False, True])
def test_ranked_screening_rescores_gathered_survivors_exactly(cuda_lib, fp8):
    """Redundant heads and a small K, ranked screening of every item: one bound
    pass keeps the keys above each row's estimate, the gathered survivors are
    scored on the tensor cores.  The selection equals the dense path's, the
    counters add up, most pairs are rejected, and no more than the oracle's
    ideal screening (threshold = the true K-th) would reject."""
    x, dtype = _redundant_heads_case(T=64, S=20000, seed=11, fp8=fp8)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    K = 32
    dense = to_numpy(Index(dtype).dense_topk(*_args(xd, K)))
    out, st = Index(dtype, screening=3).topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(out), dense)
    T, S = x["q"].shape[0], x["k"].shape[0]
    visible = sum(S - T + t + 1 for t in range(T))
    assert st["exact_pairs"] + st["rejected_pairs"] == visible
    assert st["rescored_pairs"] > 0, st
    assert st["rejected_pairs"] > 0.8 * visible, st
    ov = OracleView(x, dtype)
    kb = key_mean(ov.k)
    ideal = 0
    for t in range(T):
        p = int(ov.positions[t])
        res = certified_topk_row(ov.q[t], ov.w[t], ov.k[: p + 1], K, k_bar=kb, r=4, G=2,
                                 margin_log2=-12)
        ideal += res["ideal_rejected"]
        if t % 7 == 0:
            assert_topk_matches(to_numpy(out)[t], ov.scores(t), K, mag=ov.magnitude(t), t=t)
    assert st["rejected_pairs"] <= ideal * 1.002 + 16, (st, ideal)


def _overshoot_case(fp8):
    """Redundant heads along one direction b; random keys, plus a few keys
    along b in the warm-up region (very high scores) and a few hundred keys
    along b in the middle of the sequence (high, but below those).  The
    warm-up sample then puts the first estimate above the K-th score, pass 1
    keeps too few keys, and later passes over lower bands must find the
    middle keys."""
    g = torch.Generator().manual_seed(17)
    d, H, T, S = 128, 64, 16, 20000
    b = torch.randn(d, generator=g)
    b = b / b.norm()
    q = 3.0 * b + 0.02 * torch.randn((T, H, d), generator=g)
    w = torch.rand((T, H), generator=g) / 8
    k = torch.randn((S, d), generator=g)
    k[:6] += 8.0 * b                                  # tile 0: very high
    k[S - 200:S - 194] += 8.0 * b                     # diagonal tiles: very high
    mid = torch.randperm(S - 4000, generator=g)[:300] + 2000
    k[mid] += 4.0 * b                                 # the rest of the Top-K
    so = [[0, 0, S - T], [T, S, 0]]
    if fp8:
        from exact_certified_top_b200.workloads import _e4m3_per_token
        q8, qs = _e4m3_per_token(q)
        k8, ks = _e4m3_per_token(k)
        return dict(q=q8, q_scale=qs, w=w, k=k8, k_scale=ks, seq_offsets=so,
                    positions=torch.arange(S - T, S)), "fp8"
    return dict(q=q.to(torch.bfloat16), q_scale=None, w=w, k=k.to(torch.bfloat16),
                k_scale=None, seq_offsets=so, positions=torch.arange(S - T, S)), "bf16"


@pytest.mark.parametrize("fp8", [False, True])
def test_ranked_later_passes_recover_an_estimate_set_too_high(cuda_lib, fp8):
    x, dtype = _overshoot_case(fp8)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    K = 64
    dense = to_numpy(Index(dtype).dense_topk(*_args(xd, K)))
    out, st = Index(dtype, screening=3).topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(out), dense)
    assert st["rescreened_pairs"] > 0, st
    assert st["exact_pairs"] + st["rejected_pairs"] == st["visible_pairs"]
    assert st["rejected_pairs"] > 0.5 * st["visible_pairs"], st
    ov = OracleView(x, dtype)
    for t in range(0, 16, 3):
        assert_topk_matches(to_numpy(out)[t], ov.scores(t), K, mag=ov.magnitude(t), t=t)


def test_ranked_screening_on_a_loose_bound_keeps_every_key(cuda_lib):
    """Independent random heads (the bound is loose): ranked screening keeps
    nearly every key, gathers and scores them all, and still returns the
    dense selection; the adaptive mode hands the same rows to the filter
    scorer after its probe."""
    _, x, xd = _inputs("prefill_128k_fp8", 200, 9000, 300)
    K = 300
    dense = to_numpy(Index("fp8").dense_topk(*_args(xd, K)))
    out, st = Index("fp8", screening=3).topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(out), dense)
    assert st["rescored_pairs"] > 0.5 * st["visible_pairs"], st
    out2, st2 = Index("fp8", screening=2, probe_sample=0).topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(out2), dense)
    assert st2["rescored_pairs"] == 0 and st2["filtered_pairs"] == st2["visible_pairs"], st2


def test_probe_samples_items_first(cuda_lib):
    """Adaptive screening probes every 7th work item (longest rows first)
    before the others.  On random inputs no sampled item finds ranked
    screening worth it, so no item is screened past its probe (no screened
    pairs are counted) and the filter scorer scores every pair.  On redundant
    heads the sample finds it worth it, every item is probed, and most pairs
    are rejected.  The selection is the dense path's either way."""
    _, x, xd = _inputs("prefill_128k_fp8", 640, 6000, 300)
    K = 300
    idx = Index("fp8")
    out, st = idx.topk(*_args(xd, K), stats=True)
    assert np.array_equal(to_numpy(out), to_numpy(idx.dense_topk(*_args(xd, K))))
    assert st["screened_pairs"] == 0 and st["filtered_pairs"] == st["visible_pairs"], st
    x2, dtype = _redundant_heads_case(T=64, S=20000, seed=11, fp8=True)
    xd2 = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x2.items()}
    K2 = 32
    out2, st2 = Index(dtype).topk(*_args(xd2, K2), stats=True)
    assert np.array_equal(to_numpy(out2), to_numpy(Index(dtype).dense_topk(*_args(xd2, K2))))
    assert st2["rejected_pairs"] > st2["visible_pairs"] // 2, st2
    assert st2["rescored_pairs"] > 0, st2


@pytest.mark.parametrize("scale_log2", [-90, 60])
def test_certified_equals_dense_at_extreme_weight_magnitudes(cuda_lib, scale_log2):
    """Weights scaled by a power of two (every score scales exactly with
    them): the head sums stay in the normal fp32 range, where the doubled head
    sum of the certified and filter scorers rounds like the dense scorer's, so
    the selections are identical in every screening mode."""
    wl, x, xd = _inputs("causal_1k_bf16", 301, 2500, 100)
    xd["w"] = (xd["w"].double() * 2.0 ** scale_log2).float()
    dense = to_numpy(Index("bf16").dense_topk(*_args(xd, 100)))
    for screening in (3, 2, 1, 0):
        idx = Index("bf16", screening=screening)
        assert np.array_equal(to_numpy(idx.topk(*_args(xd, 100))), dense), screening


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_short_rows_take_the_dense_path_with_the_same_selection(cuda_lib, dtype):
    """The adaptive mode hands a call whose sequences all have at most
    short_dense_keys keys to the dense scorer and radix Top-K: the selection is
    the certified machinery's, the stats count every pair as exact."""
    base = "causal_1k_bf16" if dtype == "bf16" else "prefill_128k_fp8"
    wl, x, xd = _inputs(base, 300, 3000, 256)
    K = 256
    short, st = binding.Index(wl.dtype, short_dense_keys=4096).topk(*_args(xd, K), stats=True)
    full, st_full = Index(wl.dtype).topk(*_args(xd, K), stats=True)
    dense = binding.Index(wl.dtype).dense_topk(*_args(xd, K))
    assert torch.equal(short, dense) and torch.equal(full, dense)
    assert st["visible_pairs"] == st["exact_pairs"] == wl.visible_pairs
    assert st["screened_pairs"] == st["filtered_pairs"] == st["candidates"] == 0, st
    assert st_full["filtered_pairs"] > 0, st_full
    # above the limit the certified machinery runs
    _, st_long = binding.Index(wl.dtype, short_dense_keys=2999).topk(*_args(xd, K), stats=True)
    assert st_long["filtered_pairs"] > 0, st_long
