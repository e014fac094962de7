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
