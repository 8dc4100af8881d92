"""The multi-GPU launch of bench.py, rehearsed on CPU: two gloo ranks run the
same host-side plumbing (per-rank problems, max-over-ranks timing, the
aggregate rate, the reference arm's rank gate) that torchrun ranks run on GPUs.
"""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime

    import ag_inputs
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        base = ag_inputs.Workload("multirank_tiny", B=1, L=64, seed=5)
        w = bench.rank_workload(base, rank)
        inp = ag_inputs.make_inputs(w)
        # Every rank's q as seen by rank 0, to check the problems differ.
        qs = [torch.empty_like(inp["q"].float()) for _ in range(world)]
        dist.all_gather(qs, inp["q"].float())
        # Rank r took (r + 1) seconds: all ranks must see the slowest, 2 s.
        slowest = bench.max_over_ranks(float(rank + 1), torch.device("cpu"), world)
        rate = bench.aggregate_rate(world, 10.0, 4, slowest)
        # The reference arm runs on rank 0 only; the others return at once.
        out = io.StringIO()
        if rank != 0:
            with redirect_stdout(out):
                bench.run_reference(None, rank, world)
        results[rank] = {
            "seed": w.seed,
            "same_q_as_rank0": bool(torch.equal(qs[0], qs[rank])),
            "q_differs": not torch.equal(qs[0], qs[1]),
            "slowest": slowest,
            "rate": rate,
            "ref_output": out.getvalue(),
        }
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_follow_the_bench_protocol():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(results)
    assert sorted(res) == [0, 1]
    assert res[0]["seed"] == 5 and res[1]["seed"] == 1005      # own problem per rank
    assert res[0]["q_differs"] and res[1]["q_differs"]
    assert res[0]["same_q_as_rank0"] and not res[1]["same_q_as_rank0"]
    assert res[0]["slowest"] == pytest.approx(2.0) and res[1]["slowest"] == pytest.approx(2.0)
    # world * units * steps / slowest time: 2 * 10 * 4 / 2 s.
    assert res[0]["rate"] == pytest.approx(40.0) and res[1]["rate"] == pytest.approx(40.0)
    assert res[1]["ref_output"] == ""                              # rank 1: no work, no line


def test_single_rank_helpers():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import ag_inputs
    import bench

    base = ag_inputs.WORKLOADS["tiny"]
    assert bench.rank_workload(base, 0) == base
    assert bench.rank_workload(base, 3).seed == base.seed + 3000
    assert bench.max_over_ranks(1.5, torch.device("cpu"), 1) == 1.5
    assert bench.aggregate_rate(1, 8.0, 5, 2.0) == 20.0
