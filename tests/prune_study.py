#!/usr/bin/env python3
"""How much can the certificate prune at all?  A study on the oracle alone.

For each workload, on rows spread evenly over the positions where pruning is
possible (at least 4K visible keys), it computes with the fp64 oracle:
  * the ideal prune rate: the share of visible pairs that are non-seed keys
    whose bound plus margin lies below the row's true K-th score (the most any
    threshold schedule can reject: a threshold never exceeds the K-th), for
    retained-head budgets r in {4, 8, 16, |P|} and negative groups G in {0, 1, 2};
  * the ranked schedule's own prune rate (r = 4, G = 2, the library's default
    certificate), as the GPU runs it;
  * the two residual bounds of the certificate (the per-head Cauchy-Schwarz sum
    and the joint spectral one) and which is smaller.

    python tests/prune_study.py [--rows 64] [--out tests/golden/prune_study.json]
                                [--workloads A,B] [--merge]

--merge keeps the stored results of the workloads not listed.

Every number comes from oracle/ (the certificate, the bound, the exact scores);
the seeded generator only draws the inputs.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

from exact_certified_top_b200.workloads import WORKLOADS, codes_numpy, generate  # noqa: E402
from oracle import (certificate_setup, dequantize, indexer_scores, key_mean,  # noqa: E402
                    ranked_topk_row, seed_mask, soundness_margin, upper_bound)

STUDY_WORKLOADS = ["prefill_128k_fp8", "tight_64k_bf16_levels", "redundant_chunk128k_fp8",
                   "redundant_128k_fp8"]
BUDGETS = [4, 8, 16, "P"]
GROUPS = [0, 1, 2]
MARGIN_LOG2 = -12


def warmup_tiles(K: int) -> int:
    """The library's warm-up: enough key tiles for K exact scores, plus tile 0,
    rounded up to its threshold checkpoint interval of 4 tiles."""
    return ((K + 127) // 128 + 1 + 3) // 4 * 4


def study_rows(wl, n_rows: int) -> list:
    lo = max(0, 4096 - wl.q_pos0)
    return sorted(set(np.linspace(wl.T - 1, lo, n_rows).astype(int).tolist()))


def row_study(q, w, k, kb, K):
    n = k.shape[0]
    p = n - 1
    I = indexer_scores(q, w, k)
    vK = float(np.partition(I, n - K)[n - K])
    seeds = seed_mask(p, 64, 512)
    delta = soundness_margin(q, w, k, MARGIN_LOG2)
    out = {"visible": n, "ideal": {}}
    n_pos = int((w > 0).sum())
    for r in BUDGETS:
        rr = n_pos if r == "P" else r
        for G in GROUPS:
            cert = certificate_setup(q, w, kb, rr, G)
            ub = upper_bound(cert, q, k)
            out["ideal"][f"r={r},G={G}"] = int(np.sum(~seeds & (ub + delta < vK)))
            if r == 4 and G == 2:
                out["beta_sum"] = cert.beta_sum
                out["beta_joint"] = cert.beta_joint
    ranked = ranked_topk_row(q, w, k, K, k_bar=kb, warm_tiles=warmup_tiles(K), r=4, G=2,
                             margin_log2=MARGIN_LOG2)
    out["ranked_rejected"] = ranked["rejected"]
    out["ranked_passes"] = ranked["passes"]
    return out


def study(name: str, n_rows: int) -> dict:
    wl = WORKLOADS[name]
    t0 = time.perf_counter()
    x = generate(wl)
    ks = None if x["k_scale"] is None else x["k_scale"].numpy()
    k = dequantize(codes_numpy(x["k"]), ks, wl.dtype)
    kb = key_mean(k)
    rows = study_rows(wl, n_rows)

    def one(t):
        qs = None if x["q_scale"] is None else x["q_scale"][t:t + 1].numpy()
        q = dequantize(codes_numpy(x["q"][t:t + 1]), qs, wl.dtype)[0]
        w = x["w"][t].numpy().astype(np.float64)
        return row_study(q, w, k[: wl.q_pos0 + t + 1], kb, wl.K)

    from threadpoolctl import threadpool_limits
    with threadpool_limits(1):
        with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
            res = list(ex.map(one, rows))
    vis = sum(r["visible"] for r in res)
    ideal = {key: round(100.0 * sum(r["ideal"][key] for r in res) / vis, 3)
             for key in res[0]["ideal"]}
    bs = np.array([r["beta_sum"] for r in res])
    bj = np.array([r["beta_joint"] for r in res])
    return {
        "workload": name, "rows": rows, "visible_pairs": vis,
        "ideal_prune_pct": ideal,
        "ranked_prune_pct": round(100.0 * sum(r["ranked_rejected"] for r in res) / vis, 3),
        "ranked_rows_needing_more_passes": int(sum(r["ranked_passes"] > 1 for r in res)),
        "beta_sum_median": float(np.median(bs)), "beta_joint_median": float(np.median(bj)),
        "joint_smaller_rows": int(np.sum(bj < bs)),
        "seconds": round(time.perf_counter() - t0, 1),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=64)
    ap.add_argument("--out", default=os.path.join(HERE, "golden", "prune_study.json"))
    ap.add_argument("--workloads", default=",".join(STUDY_WORKLOADS))
    ap.add_argument("--merge", action="store_true",
                    help="keep the stored results of the workloads not listed")
    args = ap.parse_args()
    results = [study(name, args.rows) for name in args.workloads.split(",")]
    if args.merge and os.path.exists(args.out):
        with open(args.out) as f:
            stored = json.load(f)
        assert stored["rows_per_workload"] == args.rows and stored["margin_log2"] == MARGIN_LOG2
        done = {r["workload"] for r in results}
        order = {name: i for i, name in enumerate(STUDY_WORKLOADS)}
        results = sorted([r for r in stored["results"] if r["workload"] not in done] + results,
                         key=lambda r: order.get(r["workload"], len(order)))
    with open(args.out, "w") as f:
        json.dump({"margin_log2": MARGIN_LOG2, "rows_per_workload": args.rows,
                   "results": results}, f, indent=1)
    for r in results:
        print(json.dumps({k: v for k, v in r.items() if k != "rows"}))


if __name__ == "__main__":
    main()
