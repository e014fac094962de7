"""Host-side pieces of bench.py that need no GPU: the oracle's ideal prune
sample reported beside the certified line, and the config record."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_certified_top_b200.workloads import generate, small_case  # noqa: E402


def test_ideal_prune_sample_is_an_upper_limit_of_the_schedule():
    """The ideal rate (threshold = true K-th score) bounds the oracle
    schedule's rate from above; on redundant heads both are large, on the
    synthetic generator both are near zero."""
    wl = small_case("causal_1k_bf16", 32, 1200, q_pos0=1168, K=64)
    res = bench.ideal_prune_sample(generate(wl), wl, n_rows=2)
    assert 0.0 <= res["schedule_prune_pct"] <= res["ideal_prune_pct"] <= 1.0
    assert res["kind"] == "oracle"
    # redundant heads: near copies of one direction, mostly positive weights
    g = torch.Generator().manual_seed(3)
    T, S, H, d = 8, 1500, 64, 128
    q = torch.randn((T, 1, d), generator=g) + 0.02 * torch.randn((T, H, d), generator=g)
    w = torch.rand((T, H), generator=g) / 8
    x = dict(q=q.to(torch.bfloat16), q_scale=None, w=w,
             k=torch.randn((S, d), generator=g).to(torch.bfloat16), k_scale=None,
             positions=torch.arange(S - T, S))
    red = small_case("causal_1k_bf16", T, S, q_pos0=S - T, K=32)
    res = bench.ideal_prune_sample(x, red, n_rows=2)
    assert 0.0 < res["schedule_prune_pct"] <= res["ideal_prune_pct"]
    assert res["ideal_prune_pct"] > 50.0


def test_config_names_only_non_default_ablations():
    wl = small_case("causal_1k_bf16", 8, 64)
    c = bench.config_of(wl, "certified", 1, 2, "sparse", {"probe_sample": 0})
    assert c["screening"] == 2 and c["writeback"] == "sparse" and c["probe_sample"] == 0
    c = bench.config_of(wl, "dense", 2)
    assert "screening" not in c and c["parallelism"] == "rows x2"


@pytest.mark.parametrize("flag", ["--probe-sample", "--block-bound"])
def test_ablation_flags_parse(flag, monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", flag, "0"])
    args = bench.parse_args()
    assert getattr(args, flag.lstrip("-").replace("-", "_")) == 0


def test_traffic_scales_reads_by_pairs_and_writes_by_candidates(monkeypatch):
    """A split traffic record: reads per visible pair, writes per appended
    candidate, each scaled by the launch's own counts; an older record scales
    everything by pairs; a record of other sources gives none."""
    wl = small_case("prefill_128k_fp8", 8, 64)
    split = {"dram_read_bytes_per_pair": 0.25, "dram_write_bytes_per_candidate": 6.0}
    monkeypatch.setattr(bench, "_traffic_record", lambda kernel, w: split)
    assert bench._traffic_per_launch("filter", wl, 1000.0, 100.0) == 250 + 600
    assert bench._traffic_per_launch("filter", wl, 1000.0) is None      # no candidate count
    monkeypatch.setattr(bench, "_traffic_record", lambda kernel, w: {"dram_bytes_per_pair": 0.5})
    assert bench._traffic_per_launch("filter", wl, 1000.0, 100.0) == 500
    monkeypatch.setattr(bench, "_traffic_record", lambda kernel, w: None)
    assert bench._traffic_per_launch("filter", wl, 1000.0, 100.0) is None

