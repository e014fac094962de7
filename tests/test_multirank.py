"""World-size-2 gloo checks of bench.py's multi-rank plumbing on CPU: the
step time is the max over ranks, every rank draws its own sequence, the job
value counts every rank's pairs, and only rank 0 runs the reference arm."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    from exact_certified_top_b200.workloads import WORKLOADS, generate, small_case
    step_ms = 10.0 * (rank + 1)                       # rank 1 is the slow one
    ms = bench.max_over_ranks(step_ms, world)
    wl = bench.rank_workload(small_case("causal_1k_bf16", 8, 64), rank)
    x = generate(wl)
    value = bench.job_value(wl.visible_pairs, world, ms)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, ms, wl.seed, float(x["k"].float().sum()), value, wl.visible_pairs))


def test_two_gloo_ranks_max_time_and_independent_sequences():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, seed0, k0, v0, pairs), (r1, ms1, seed1, k1, v1, _) = res
    assert ms0 == ms1 == 20.0                         # max over ranks
    assert seed0 != seed1 and k0 != k1                # independent sequences
    assert v0 == v1 == pytest.approx(2 * pairs / 0.020)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "causal_1k_bf16"
        tail_rows = 0
        steps = 1
        warmup = 0
    bench.run_reference(Args(), world=2, rank=1)
    assert capsys.readouterr().out == ""


def _split_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    from exact_certified_top_b200.workloads import generate, small_case
    from oracle import dense_topk
    from parity import OracleView
    wl = small_case("causal_1k_bf16", 90, 90, K=16)
    x = generate(wl)
    ov = OracleView(x, wl.dtype)
    blocks_all = bench.zigzag_blocks(wl.T, world)
    # this rank's rows only (the selection stands in for the library call)
    local = [dense_topk(ov.q, ov.w, ov.k, ov.positions, wl.K, rows=range(r0, r1))
             for r0, r1 in blocks_all[rank]]
    local = torch.as_tensor(__import__("numpy").concatenate(local), dtype=torch.int32)
    full = bench.gather_rows(local, blocks_all, wl.T)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, full.numpy(), bench.block_pairs(blocks_all[rank], wl.q_pos0)))


def test_two_gloo_ranks_split_one_sequence_by_rows():
    """--split rows: the rows of one sequence in zigzag blocks over 2 ranks;
    every rank ends with the full selection, equal to one rank's result."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from exact_certified_top_b200.workloads import generate, small_case
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import dense_topk
    from parity import OracleView
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = small_case("causal_1k_bf16", 90, 90, K=16)
    ov = OracleView(generate(wl), wl.dtype)
    want = dense_topk(ov.q, ov.w, ov.k, ov.positions, wl.K)
    for _, full, _ in res:
        assert np.array_equal(full, want)
    p0, p1 = res[0][2], res[1][2]
    assert p0 + p1 == wl.visible_pairs
    assert abs(p0 - p1) <= 0.05 * max(p0, p1)


@pytest.mark.parametrize("T,world", [(131072, 8), (131072, 2), (8192, 4), (1000, 3), (90, 2),
                                     (16384, 7)])
def test_zigzag_blocks_cover_every_row_once_and_balance_causal_pairs(T, world):
    sys.path.insert(0, ROOT)
    import bench
    blocks = bench.zigzag_blocks(T, world)
    rows = sorted(r for b in blocks for r0, r1 in b for r in range(r0, r1))
    assert rows == list(range(T))
    pairs = [bench.block_pairs(b, 0) for b in blocks]
    assert sum(pairs) == T * (T + 1) // 2
    # a rank's share differs from the mean by at most a block's rows times T
    mean = sum(pairs) / world
    assert max(abs(p - mean) for p in pairs) <= (T / (2 * world) + 1) * 2 + 0.01 * mean
