#!/usr/bin/env python3
"""Throughput of the DoSA indexer Top-K on B200s (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--path certified|dense]

A step is one pass of the whole indexer (every row of the workload through
the library's Top-K call) over inputs already resident in HBM.  The headline
workload is 128K-token causal prefill with fp8 e4m3 inputs, H = 64, d = 128,
K = 2048.  With N > 1 (torchrun) every rank processes its own independent
sequence of the same shape (weak scaling, no collective on the data path), or
with --split rows the ranks share one sequence: its query rows are cut into 2N
blocks, rank i scores blocks i and 2N-1-i (every rank gets the same number of
causal pairs to within a block's worth), the keys are replicated, and the
selected indices are all-gathered (strong scaling).  The step time is the max
over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_certified_top_b200.workloads import WORKLOADS, generate  # noqa: E402

METRIC = "indexer query·key pairs/sec @128K causal, K=2048 (1 B200); prune %; % roofline"
UNIT = "pairs/s"
L2_FLUSH_BYTES = 256 << 20          # twice the 126 MB L2


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_128k_fp8", choices=sorted(WORKLOADS))
    ap.add_argument("--path", choices=["certified", "dense", "scorer", "decode"],
                    default="certified",
                    help="dense: dense scorer + Top-K; scorer: the dense scorer alone (every "
                         "visible score written, no Top-K); decode: the decode-step call on a "
                         "decode workload (decode_1m_fp8)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the oracle CPU baseline sample")
    ap.add_argument("--screening", type=int, choices=[0, 1, 2, 3], default=2,
                    help="certified path: 0 no bounds, 1 streaming schedule (every tile), "
                         "2 adaptive (default), 3 ranked schedule for every item")
    ap.add_argument("--block-bound", type=int, choices=[0, 1], default=1,
                    help="certified path: skip key tiles whose key-block bound rules them out")
    ap.add_argument("--probe-sample", type=int, choices=[0, 1], default=1,
                    help="adaptive screening: probe every 7th work item first (1) or every item (0)")
    ap.add_argument("--short-dense-keys", type=int, default=16384,
                    help="adaptive screening: calls whose sequences all have at most this many "
                         "keys take the dense scorer and Top-K (0: never)")
    ap.add_argument("--writeback", choices=["sparse", "dense"], default="sparse",
                    help="certified path: packed candidates >= threshold (default), or every "
                         "exact score into a dense matrix and its dense Top-K (ablation)")
    ap.add_argument("--tail-rows", type=int, default=0,
                    help="profile only the last N query rows of the workload (same keys)")
    ap.add_argument("--split", choices=["sequences", "rows"], default="sequences",
                    help="N > 1: an independent sequence per rank (default), or the rows of one "
                         "sequence in causal-balanced zigzag blocks with the indices all-gathered")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing

def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Max of a host scalar over all ranks (step times: the slowest rank)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(wl, rank: int):
    """Each rank runs its own independent sequence of the workload's shape."""
    from dataclasses import replace
    return replace(wl, seed=wl.seed + rank)


def job_value(pairs_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job pairs/s: every rank's pairs over the slowest rank's step time."""
    return world * pairs_per_rank / (ms_per_step_max * 1e-3)


def zigzag_blocks(T: int, world: int) -> list:
    """Rows [0, T) of one causal sequence cut into 2 * world contiguous blocks;
    rank i takes blocks i and 2 * world - 1 - i, a short block and a long one,
    so every rank scores about the same number of causal pairs.  Returns, per
    rank, its two (first row, end row) ranges."""
    n = 2 * world
    edges = [T * j // n for j in range(n + 1)]
    return [[(edges[i], edges[i + 1]), (edges[n - 1 - i], edges[n - i])] for i in range(world)]


def block_pairs(blocks, q_pos0: int) -> int:
    """Visible causal pairs of a rank's row ranges (row t sits at q_pos0 + t)."""
    return sum((r1 - r0) * (2 * q_pos0 + r0 + r1 + 1) // 2 for r0, r1 in blocks)


def gather_rows(local: torch.Tensor, blocks_all: list, T: int) -> torch.Tensor:
    """All-gather every rank's selected indices (its rows, in block order) into
    the full [T, K] result on every rank."""
    world = len(blocks_all)
    n_max = max(sum(r1 - r0 for r0, r1 in b) for b in blocks_all)
    K = local.shape[1]
    pad = torch.full((n_max, K), -1, dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    torch.distributed.all_gather(parts, pad)
    full = torch.empty((T, K), dtype=local.dtype, device=local.device)
    for part, blocks in zip(parts, blocks_all):
        at = 0
        for r0, r1 in blocks:
            full[r0:r1] = part[at: at + r1 - r0]
            at += r1 - r0
    return full


# ---------------------------------------------------------------------------
# clocks during the timed region

CLOCK_FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
                "clocks_event_reasons.active", "clocks_event_reasons.hw_slowdown",
                "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


def clocks_start(local_rank):
    path = tempfile.mktemp(prefix="dosa_clocks_", suffix=".csv")
    try:
        f = open(path, "w")
        p = subprocess.Popen(["nvidia-smi", "-i", str(local_rank),
                              "--query-gpu=" + ",".join(CLOCK_FIELDS),
                              "--format=csv,noheader,nounits", "-lms", "200"],
                             stdout=f, stderr=subprocess.DEVNULL)
        return p, f, path
    except (OSError, FileNotFoundError) as e:
        print(f"clock sampling unavailable: {e}", file=sys.stderr)
        return None


def clocks_stop(handle):
    if handle is None:
        return None
    p, f, path = handle
    p.terminate()
    try:
        p.wait(timeout=5)
    except subprocess.TimeoutExpired:
        p.kill()
    f.close()
    rows = []
    with open(path) as fh:
        for line in fh:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == len(CLOCK_FIELDS):
                rows.append(parts)
    os.unlink(path)
    if not rows:
        return None

    def num(x):
        try:
            return float(x)
        except ValueError:
            return float("nan")
    loaded = [r for r in rows if num(r[4]) >= 50] or rows
    reasons = set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in loaded:
        for n, v in zip(names, r[6:10]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(num(r[1]) for r in loaded),
            "sm_max_mhz": max(num(r[2]) for r in rows),
            "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded),
            "power_w_max": max(num(r[3]) for r in rows)}


# ---------------------------------------------------------------------------
# roofline

KERNELS_PER_RECORD = {"decode": 3}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def roofline(prof: dict, wl, pairs_per_step: int, steps: int, dtype: str, stats=None):
    """Dominant kernel of the step against the tensor-core peak of its dtype.

    Algorithmic work: the dense scorer does 2*H*d flops per visible pair; the
    filter scorer 2*H*d per pair it scores; the certified kernel 2*H*d per
    exactly scored pair plus 2*d*8 per screened pair (the bound GEMM's dot
    products).  Pair counts come from the call's own counters (one untimed
    call of the same workload)."""
    peaks, src = measured_peaks()
    kernels = {k: v for k, v in prof.items() if v[0] > 0}
    if not kernels:
        return None
    dom = max(kernels, key=lambda k: kernels[k][1])
    launches, ms = kernels[dom]
    flops_per_pair = 2 * wl.H * wl.d
    # bf16 sustained peak (the kernel runs inside a long step); fp8 = 2x (nominal ratio)
    peak = peaks["bf16_tflops_sustained"] * (2.0 if dtype == "fp8" else 1.0)
    peak_src = (f"{src}: bf16_tflops_sustained"
                + (" x2 (fp8/bf16 nominal ratio)" if dtype == "fp8" else ""))
    if dom == "score":
        work = flops_per_pair * pairs_per_step * steps          # every visible pair, once
        name = "score_tc"
    elif dom == "filter" and stats:
        work = flops_per_pair * stats["filtered_pairs"] * steps
        name = "filter_kernel"
    elif dom == "certified" and stats:
        exact = stats["exact_pairs"] - stats.get("filtered_pairs", 0)
        work = (flops_per_pair * exact + 2 * wl.d * 8 * stats["screened_pairs"]) * steps
        name = "certified_kernel"
    elif dom == "rescore" and stats:
        work = flops_per_pair * stats["rescored_pairs"] * steps
        name = "rescore_kernel"
    elif dom == "rank" and stats:
        # the bound pass is bound by its epilogue's fp32 ALU work: 18 operations
        # per screened pair (4 ReLU + 4 multiply-adds of the retained heads, the
        # norm term, 2 x (2 multiply-adds, a ReLU, a subtraction) of the negative
        # aggregates, the scale product), one operation per FP32 lane per clock
        clk = (measured_peaks()[0].get("sm_max_mhz") or 1965.0) * 1e6
        alu_peak = 148 * 128 * clk / 1e12              # T ops/s
        ops = 18 * (stats["screened_pairs"] + stats.get("rescreened_pairs", 0)) * steps
        achieved = ops / (ms * 1e-3) / 1e12
        return {"kernel": "rank_screen_kernel (+ rank_prep)", "bound": "alu",
                "achieved": round(achieved, 2), "peak": round(alu_peak, 2), "unit": "Tops/s",
                "frac": round(achieved / alu_peak, 4), "traffic": None,
                "peak_source": "148 SMs x 128 FP32 lanes x sm_max_mhz (one op per lane per clock)",
                "launches": launches, "avg_launch_ms": round(ms / launches, 3)}
    elif dom == "decode" and stats:
        # seed + split-S scan + finish: every visible pair scored on the tensor
        # cores, every key of the cache read once per call.  The bound is the
        # slower of the two ideal times.
        kbytes = wl.S * wl.d * (1 if dtype == "fp8" else 2) + (wl.S * 4 if dtype == "fp8" else 0)
        flops = flops_per_pair * stats["exact_pairs"]
        t_tensor = flops / (peak * 1e12)
        t_hbm = kbytes / (peaks["hbm_gbs"] * 1e9)
        avg = ms / launches
        traffic = _traffic_record("decode", wl)
        traffic = None if traffic is None else round(traffic["dram_bytes_per_launch"])
        if t_hbm >= t_tensor:
            achieved = kbytes / (avg * 1e-3) / 1e9
            return {"kernel": "decode_seed+decode_scan+decode_finish", "bound": "hbm",
                    "achieved": round(achieved, 1), "peak": round(peaks["hbm_gbs"], 1),
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": traffic, "peak_source": f"{src}: hbm_gbs",
                    "launches": launches, "avg_launch_ms": round(avg, 4)}
        achieved = flops / (avg * 1e-3) / 1e12
        return {"kernel": "decode_seed+decode_scan+decode_finish", "bound": "tensor",
                "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_src,
                "launches": launches, "avg_launch_ms": round(avg, 4)}
    else:
        return {"kernel": dom, "launches": launches, "avg_launch_ms": round(ms / launches, 3)}
    achieved = work / (ms * 1e-3) / 1e12
    return {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1),
            "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "traffic": _traffic_per_launch(
                dom, wl, pairs_per_step * steps / launches,
                stats["candidates"] * steps / launches if stats else None),
            "peak_source": peak_src, "launches": launches,
            "avg_launch_ms": round(ms / launches, 3)}


def _traffic_record(kernel: str, wl):
    """The committed ncu DRAM-traffic record of a kernel, or None when there is
    none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(f"{kernel}:{wl.dtype}")
    if not rec or rec.get("source_sha") != _kernel_source_sha(kernel):
        return None
    return rec


def _traffic_per_launch(kernel: str, wl, pairs_per_launch: float, cands_per_launch=None):
    """DRAM bytes per launch from a committed ncu summary: the reads scaled by
    the launch's visible pairs (queries, keys, scales), the writes by its
    appended candidates (8-byte packed entries), each from the capture's own
    ratio; or, for an older record, all bytes scaled by pairs."""
    rec = _traffic_record(kernel, wl)
    if rec is None:
        return None
    if "dram_read_bytes_per_pair" in rec and cands_per_launch is not None:
        return round(rec["dram_read_bytes_per_pair"] * pairs_per_launch
                     + rec["dram_write_bytes_per_candidate"] * cands_per_launch)
    if "dram_bytes_per_pair" not in rec:
        return None
    return round(rec["dram_bytes_per_pair"] * pairs_per_launch)


# The sources a kernel's traffic record was taken from: its own file and the
# headers it includes.
KERNEL_SOURCES = {
    "filter": ("filter.cu", "cand_state.cuh", "dosa_device.cuh", "dosa_internal.h",
               "score_epilogue.cuh", "work_items.cuh"),
    "decode": ("decode.cu", "cand_state.cuh", "dosa_device.cuh", "dosa_internal.h",
               "score_epilogue.cuh", "work_items.cuh"),
}


def _kernel_source_sha(kernel: str):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "exact_certified_top_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of rows

def oracle_sample(x, wl, budget_s: float):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import dense_topk, dequantize
    from exact_certified_top_b200.workloads import codes_numpy
    from threadpoolctl import threadpool_info
    # rows spread evenly over the workload, visited in an interleaved order
    # bit-reversal order over 1024 evenly spaced rows: any prefix is spread out
    n_s = min(1024, wl.T)
    base = np.linspace(0, wl.T - 1, n_s).astype(np.int64)
    bits = max(1, int(np.ceil(np.log2(n_s))))
    rev = [int(format(i, f"0{bits}b")[::-1], 2) for i in range(1 << bits)]
    order = base[[r for r in rev if r < n_s]]
    kscale = None if x["k_scale"] is None else x["k_scale"].cpu().numpy()
    k = dequantize(codes_numpy(x["k"]), kscale, wl.dtype)
    pos = x["positions"].cpu().numpy()
    done, pairs = [], 0
    t0 = time.perf_counter()
    for t in order:
        q_t = x["q"][t:t + 1]
        qs = None if x["q_scale"] is None else x["q_scale"][t:t + 1].cpu().numpy()
        q = dequantize(codes_numpy(q_t), qs, wl.dtype)
        w = x["w"][t:t + 1].cpu().numpy().astype(np.float64)
        dense_topk(q, w, k, pos[t:t + 1], wl.K)
        done.append(int(t))
        pairs += int(pos[t]) + 1
        if time.perf_counter() - t0 > budget_s and len(done) >= 2:
            break
    el = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": pairs / el, "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "sample": f"{len(done)} rows of {wl.name} spread evenly over positions "
                      f"(pairs {pairs}), fp64 dense scoring + full sort, {el:.1f} s",
            "host_cores": os.cpu_count()}


def ideal_prune_sample(x, wl, n_rows: int = 64):
    """The certificate's ideal prune rate (the oracle's: threshold equal to
    the true K-th score, the default certificate r = 4, G = 2) and the
    oracle schedule's own prune rate, on n_rows rows spread over the
    workload's positions (the longest first), one row per host core at a
    time; plus the committed oracle prune study's figure for the workload
    (tests/golden/prune_study.json, written by tests/prune_study.py) when it
    has one."""
    from concurrent.futures import ThreadPoolExecutor
    from threadpoolctl import threadpool_limits
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import certified_topk_row, dequantize, key_mean
    from exact_certified_top_b200.workloads import codes_numpy
    kscale = None if x["k_scale"] is None else x["k_scale"].cpu().numpy()
    k = dequantize(codes_numpy(x["k"]), kscale, wl.dtype)
    kb = key_mean(k)
    pos = x["positions"].cpu().numpy()
    rows = sorted({int(r) for r in np.linspace(wl.T - 1, 0, n_rows + 1)[:n_rows]}, reverse=True)
    qc = codes_numpy(x["q"])
    qsc = None if x["q_scale"] is None else x["q_scale"].cpu().numpy()
    wv = x["w"].cpu().numpy().astype(np.float64)
    t0 = time.perf_counter()

    def one(t):
        q = dequantize(qc[t:t + 1], None if qsc is None else qsc[t:t + 1], wl.dtype)[0]
        res = certified_topk_row(q, wv[t], k[:int(pos[t]) + 1], wl.K, k_bar=kb, r=4, G=2,
                                 margin_log2=-12)
        return res["visible"], res["ideal_rejected"], res["rejected"]

    with threadpool_limits(1):
        with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
            out = list(ex.map(one, rows))
    vis = sum(o[0] for o in out)
    ideal = sum(o[1] for o in out)
    rej = sum(o[2] for o in out)
    res = {"ideal_prune_pct": round(100.0 * ideal / max(vis, 1), 4),
           "schedule_prune_pct": round(100.0 * rej / max(vis, 1), 4), "kind": "oracle",
           "sample": f"{len(rows)} rows of {wl.name} spread over its positions ({vis} visible "
                     f"pairs), {time.perf_counter() - t0:.1f} s"}
    study = os.path.join(ROOT, "tests", "golden", "prune_study.json")
    if os.path.exists(study):
        with open(study) as f:
            for r in json.load(f)["results"]:
                if r["workload"] == wl.name:
                    res["study"] = {"file": "tests/golden/prune_study.json",
                                    "rows": len(r["rows"]),
                                    "ideal_prune_pct": r["ideal_prune_pct"],
                                    "ranked_prune_pct": r.get("ranked_prune_pct")}
    return res


# ---------------------------------------------------------------------------

def ablations_of(args) -> dict:
    """Certified-path switches that differ from their defaults."""
    if args.path != "certified":
        return {}
    defaults = {"block_bound": 1, "probe_sample": 1, "short_dense_keys": 16384}
    return {k: getattr(args, k) for k, v in defaults.items() if getattr(args, k) != v}


def config_of(wl, path, world, screening=None, writeback=None, ablations=None):
    extra = {"screening": screening} if screening is not None else {}
    if writeback is not None:
        extra["writeback"] = writeback
    extra.update(ablations or {})
    # world < 0: the rows of one sequence split over -world ranks (zigzag)
    par = f"rows zigzag x{-world}, indices all-gathered" if world < 0 else f"rows x{world}"
    return {"workload": wl.name, "T": wl.T, "S": wl.S, "H": wl.H, "d": wl.d, "K": wl.K,
            "dtype": wl.dtype, "q_pos0": wl.q_pos0, "path": path, **extra,
            "parallelism": par,
            "l2": "flushed between timed steps (256 MiB write, outside the timed windows)",
            "visible_pairs_per_gpu": wl.visible_pairs}


def run_reference(args, world, rank):
    if rank != 0:
        return
    wl = workload_of(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = generate(wl, device=dev)
    per_step = max(2.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(x, wl, per_step / 4)
    vals = []
    last = None
    for _ in range(args.steps):
        last = oracle_sample(x, wl, per_step)
        vals.append(last["value"])
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, "oracle", world),
            "cpu_baseline": {**last, "value": v},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_of(args):
    wl = WORKLOADS[args.workload]
    if args.tail_rows:
        from dataclasses import replace
        n = min(args.tail_rows, wl.T)
        wl = replace(wl, name=f"{wl.name}[last {n} rows]", T=n, q_pos0=wl.q_pos0 + wl.T - n)
    return wl


def run_ours(args, world, rank, local):
    from exact_certified_top_b200 import binding
    binding.load()
    wl = workload_of(args)
    split_rows = world > 1 and args.split == "rows"
    if split_rows and args.path not in ("certified", "dense"):
        raise SystemExit("--split rows runs the certified or the dense path")
    # one shared sequence (same seed on every rank) or one per rank
    x = generate(wl if split_rows else rank_workload(wl, rank), device="cuda")
    idx = binding.Index(wl.dtype, H=wl.H, max_K=max(2048, wl.K), screening=args.screening,
                        sparse_writeback=int(args.writeback == "sparse"),
                        block_bound=args.block_bound, probe_sample=args.probe_sample,
                        short_dense_keys=args.short_dense_keys)
    certified = args.path == "certified"
    decode = args.path == "decode"
    scorer = args.path == "scorer"
    if decode and wl.decode_noise <= 0:
        raise SystemExit("--path decode needs a decode workload (decode_1m_fp8)")
    seeds = None
    if wl.decode_noise > 0:
        # decode workload: row 0 is the previous step, rows 1.. are timed; the
        # previous step's selection (dense, untimed) seeds the decode call
        from dataclasses import replace
        m = wl.T - 1
        one = lambda v: None if v is None else v[:1]
        rest = lambda v: None if v is None else v[1:]
        prev_so = [[0, 0, wl.q_pos0], [1, wl.S, 0]]
        seeds = idx.dense_topk(one(x["q"]), one(x["q_scale"]), one(x["w"]), x["k"], x["k_scale"],
                               prev_so, wl.K).expand(m, wl.K).contiguous()
        x = {**x, "q": rest(x["q"]), "q_scale": rest(x["q_scale"]), "w": rest(x["w"]),
             "positions": rest(x["positions"]), "seq_offsets": [[0, 0, wl.q_pos0 + 1], [m, wl.S, 0]]}
        wl = replace(wl, name=f"{wl.name}[rows 1..{m}]", T=m, q_pos0=wl.q_pos0 + 1)
    so = x["seq_offsets"]
    blocks_all = zigzag_blocks(wl.T, world) if split_rows else None
    my_rows = (sum(r1 - r0 for r0, r1 in blocks_all[rank]) if split_rows else wl.T)
    if decode:
        ws = torch.zeros(idx.decode_workspace_size(wl.T, wl.S, wl.K), dtype=torch.uint8,
                         device="cuda")
    else:
        ws = torch.zeros(idx.workspace_size(my_rows, wl.S, wl.K, certified), dtype=torch.uint8,
                         device="cuda")
    out = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    out_local = torch.empty((my_rows, wl.K), dtype=torch.int32, device="cuda")
    call_args = (x["q"], x["q_scale"], x["w"], x["k"], x["k_scale"], so, wl.K)
    if scorer:
        # the dense scorer alone: every visible score of a chunk of rows written
        # into one fp32 matrix (about 4 GiB), chunk after chunk
        sc_rows = max(8, min(wl.T, (4 << 30) // (4 * wl.S)) // 8 * 8)
        sc_buf = torch.empty((sc_rows, wl.S), dtype=torch.float32, device="cuda")
        sc_err = torch.zeros(16, dtype=torch.uint8, device="cuda")

    def step_rows():
        # this rank's two row blocks of the shared sequence, then the exchange
        at = 0
        for r0, r1 in blocks_all[rank]:
            n = r1 - r0
            sl = lambda v: None if v is None else v[r0:r1]
            a = (sl(x["q"]), sl(x["q_scale"]), sl(x["w"]), x["k"], x["k_scale"],
                 [[0, 0, wl.q_pos0 + r0], [n, wl.S, 0]], wl.K)
            if certified:
                idx.topk(*a, out=out_local[at:at + n], workspace=ws)
            else:
                idx.dense_topk(*a, out=out_local[at:at + n], workspace=ws)
            at += n
        out.copy_(gather_rows(out_local, blocks_all, wl.T))

    def step(o=out, a=call_args):
        if split_rows:
            step_rows()
        elif scorer:
            for r0 in range(0, wl.T, sc_rows):
                n = min(sc_rows, wl.T - r0)
                idx.scores(a[0], a[1], a[2], a[3], a[4], r0, n, wl.q_pos0 + r0, wl.S, sc_buf,
                           wl.S, sc_err)
        elif decode:
            idx.decode_topk(*a, seeds, out=o, workspace=ws)
        elif certified:
            idx.topk(*a, out=o, workspace=ws)
        else:
            idx.dense_topk(*a, out=o, workspace=ws)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    binding.check_device(ws)

    # timed region: per-step CUDA events, L2 flushed between steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clk = clocks_start(local)
    binding.profile_enable(True)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        starts[i].record()
        step()
        ends[i].record()
    torch.cuda.synchronize()
    barrier(world)
    prof = binding.profile_read()
    binding.profile_enable(False)
    clocks = clocks_stop(clk)
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    ms = max_over_ranks(ms, world)
    binding.check_device(ws)

    pairs = wl.visible_pairs
    # split rows: the ranks share one sequence; otherwise each has its own
    value = job_value(pairs, 1 if split_rows else world, ms)
    # a "decode" profile record spans three kernels (seed, scan, finish)
    launches = sum(n * KERNELS_PER_RECORD.get(k, 1) for k, (n, _) in prof.items())

    stats = None
    if certified and not split_rows:
        _, stats = idx.topk(*call_args, out=out, workspace=ws, stats=True)
    elif decode:
        _, stats = idx.decode_topk(*call_args, seeds, out=out, workspace=ws, stats=True)

    # end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e and not scorer and not split_rows:
        host = {k: (v.cpu().pin_memory() if torch.is_tensor(v) and v.is_cuda else v)
                for k, v in x.items()}
        names = ["q", "q_scale", "w", "k", "k_scale"]
        h2d = sum(host[n].numel() * host[n].element_size() for n in names if host[n] is not None)
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        d2h = out_host.numel() * out_host.element_size()
        if decode:
            # the step's inputs are the new rows (q, its scales, w) and the
            # seeds; the key cache stays resident, as in serving
            names = ["q", "q_scale", "w"]
            h2d = sum(host[n].numel() * host[n].element_size() for n in names
                      if host[n] is not None) + seeds.numel() * 4
            dev_in = {n: (torch.empty_like(x[n]) if x[n] is not None else None) for n in names}
            seeds_host = seeds.cpu().pin_memory()
            seeds_dev = torch.empty_like(seeds)

            def e2e_step():
                for n in names:
                    if host[n] is not None:
                        dev_in[n].copy_(host[n], non_blocking=True)
                seeds_dev.copy_(seeds_host, non_blocking=True)
                idx.decode_topk(dev_in["q"], dev_in["q_scale"], dev_in["w"], x["k"], x["k_scale"],
                                so, wl.K, seeds_dev, out=out, workspace=ws)
                out_host.copy_(out, non_blocking=True)
        elif certified:
            # the host-staged call: query chunks stream through two device slots,
            # copies overlapping the kernels
            sot = torch.as_tensor(so, dtype=torch.int64)
            S_max = int((sot[1:, 1] - sot[:-1, 1]).max())
            hws = torch.zeros(idx.host_workspace_size(wl.T, int(sot[-1, 1]), S_max, wl.K),
                              dtype=torch.uint8, device="cuda")

            def e2e_step():
                idx.topk_host(host["q"], host["q_scale"], host["w"], host["k"], host["k_scale"],
                              so, wl.K, out=out_host, workspace=hws)
        else:
            dev_in = {n: (torch.empty_like(x[n]) if x[n] is not None else None) for n in names}

            def e2e_step():
                for n in names:
                    if host[n] is not None:
                        dev_in[n].copy_(host[n], non_blocking=True)
                a = (dev_in["q"], dev_in["q_scale"], dev_in["w"], dev_in["k"], dev_in["k_scale"],
                     so, wl.K)
                step(out, a)
                out_host.copy_(out, non_blocking=True)
        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        n_e2e = max(1, min(args.steps, 3))
        for _ in range(n_e2e):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        e2e = {"value": world * pairs / (ems * 1e-3), "unit": UNIT, "ms_per_step": round(ems, 3),
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = ideal = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not scorer:
        cpu = oracle_sample(x, wl, args.cpu_seconds)
        if certified:
            ideal = ideal_prune_sample(x, wl)

    if rank == 0:
        roof = roofline(prof, wl, pairs, args.steps, wl.dtype, stats)
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
                "higher_is_better": True, "scaling": "strong" if split_rows else "weak",
                "vs_baseline": None,
                "dtype": wl.dtype, "data": "synthetic (seeded low-rank + sink generator)",
                "config": config_of(wl, args.path, world if not split_rows else -world,
                                    args.screening if args.path == "certified" else None,
                                    args.writeback if args.path == "certified" else None,
                                    ablations_of(args)),
                "roofline": roof,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "kernels": {k: {"launches": n, "ms": round(t, 3)} for k, t in
                            ((k, v[1]) for k, v in prof.items()) for n in [prof[k][0]] if n},
                "clocks": clocks}
        if stats:
            vis = stats["visible_pairs"]
            line["prune_pct"] = round(100.0 * stats["rejected_pairs"] / vis, 3) if vis else None
            line["stats"] = stats
        if ideal:
            line["ideal_prune"] = ideal
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_init(args)
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
