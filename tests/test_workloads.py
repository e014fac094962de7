"""Host checks of the seeded input generator (no indexer arithmetic here)."""
import numpy as np
import torch

from exact_certified_top_b200.workloads import WORKLOADS, generate, small_case, codes_numpy
from oracle import decode_bf16, decode_e4m3


def test_named_workloads_and_pairs():
    assert set(WORKLOADS) == {"causal_1k_bf16", "causal_16k_bf16", "prefill_128k_fp8",
                              "prefill_128k_fp8_h32", "chunk_1m_fp8", "tight_64k_bf16_levels",
                              "decode_1m_fp8", "redundant_chunk128k_fp8", "redundant_128k_fp8"}
    assert WORKLOADS["prefill_128k_fp8_h32"].H == 32
    assert WORKLOADS["decode_1m_fp8"].visible_pairs == sum(1048576 - 5 + i + 1 for i in range(5))
    assert WORKLOADS["prefill_128k_fp8"].visible_pairs == 8_590_000_128
    assert WORKLOADS["causal_16k_bf16"].visible_pairs == 134_225_920
    assert WORKLOADS["chunk_1m_fp8"].visible_pairs == 8_556_384_256
    assert WORKLOADS["tight_64k_bf16_levels"].visible_pairs == 2_147_516_416
    assert WORKLOADS["redundant_128k_fp8"].visible_pairs == 8_590_000_128
    assert WORKLOADS["redundant_chunk128k_fp8"].visible_pairs == sum(
        131072 - 8192 + i + 1 for i in range(8192))


def test_deterministic_and_shapes():
    wl = small_case("causal_1k_bf16", 64)
    a, b = generate(wl), generate(wl)
    assert a["q"].shape == (64, 64, 128) and a["k"].shape == (64, 128) and a["w"].shape == (64, 64)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["k"], b["k"]) and torch.equal(a["w"], b["w"])
    assert a["q"].dtype == torch.bfloat16 and a["q_scale"] is None
    h32 = generate(small_case("prefill_128k_fp8_h32", 16))
    assert h32["q"].shape == (16, 32, 128) and h32["w"].shape == (16, 32)


def test_fp8_codes_finite_and_scale_absmax():
    wl = small_case("prefill_128k_fp8", 32)
    x = generate(wl)
    qc = codes_numpy(x["q"])
    assert qc.dtype == np.uint8 and not np.any((qc & 0x7F) == 0x7F)
    v = decode_e4m3(qc.reshape(32, -1))
    assert np.all(np.abs(v).max(axis=1) <= 448.0) and np.all(np.abs(v).max(axis=1) >= 416.0)
    assert x["k_scale"].shape == (32,) and torch.all(x["k_scale"] > 0)


def test_levels_case_is_integer_levels_and_half_negative():
    wl = small_case("tight_64k_bf16_levels", 48)
    x = generate(wl)
    q = decode_bf16(codes_numpy(x["q"]))
    k = decode_bf16(codes_numpy(x["k"]))
    w = x["w"].numpy().astype(np.float64)
    for arr in (q, k, w):
        nz = np.abs(arr[arr != 0])
        step = nz.min()
        lv = arr / step
        assert np.all(lv == np.round(lv)) and lv.min() >= -4 and lv.max() <= 3
        assert np.log2(step) == np.round(np.log2(step))
    assert bool(torch.all((x["w"] <= 0).sum(dim=1) >= 32))


def test_sinks_are_about_one_percent():
    wl = small_case("causal_16k_bf16", 64, 16384)
    x = generate(wl)
    frac = float(x["sinks"].float().mean())
    assert 0.007 < frac < 0.013


def test_redundant_heads_share_their_direction():
    """Heads of one query are near copies (per-head noise 0.05 per coordinate
    on a query of norm ~11), a quarter of each query's weights is negative."""
    wl = small_case("redundant_128k_fp8", 16)
    x = generate(wl)
    q = decode_e4m3(codes_numpy(x["q"])).reshape(16, 64, 128)
    qn = q / np.linalg.norm(q, axis=2, keepdims=True)
    cos = np.einsum("thd,tgd->thg", qn, qn)
    assert cos.min() > 0.95
    other = np.einsum("hd,gd->hg", qn[0], qn[1])
    assert other.max() < 0.99
    assert bool(torch.all((x["w"] < 0).sum(dim=1) == 16))
