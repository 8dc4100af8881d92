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


def _shard_worker(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime

    import ag_inputs
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        L = 160
        inp = ag_inputs.random_case(2, 8, L, 128, 128, 16, seed=9, batched_bias=True)
        # Keys and values arrive as contiguous sequence shards, one per rank.
        k0, k1 = L * rank // world, L * (rank + 1) // world
        k_full = bench.gather_keys(inp["k"][:, k0:k1].contiguous(), world)
        v_full = bench.gather_keys(inp["v"][:, k0:k1].contiguous(), world)
        q0, q1 = bench.query_shard(L, world, rank)
        slab = bench.bias_rows(inp["bias"], q0, q1)
        # Local query i of the slab must read the bias row of position q0 + i.
        rows_ok = all(torch.equal(slab[:, :, i // 16], inp["bias"][:, :, (q0 + i) // 16])
                      for i in range(q1 - q0))
        results[rank] = {"k": torch.equal(k_full, inp["k"]), "v": torch.equal(v_full, inp["v"]),
                         "range": (q0, q1), "rows_ok": rows_ok,
                         "slab_rows": slab.shape[2]}
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_query_sharding_partition_gather_and_bias_rows():
    """--shard queries on two gloo ranks: the query ranges partition [0, L) in
    multiples of 32 positions, one all_gather rebuilds every key and value in
    sequence order, and each rank's bias slab puts the row of position q0 + i
    at local row i / 16."""
    world, port = 2, _free_port()
    results = mp.Manager().dict()
    mp.spawn(_shard_worker, args=(world, port, results), nprocs=world, join=True)
    got = [results[r] for r in range(world)]
    assert all(g["k"] and g["v"] and g["rows_ok"] for g in got)
    ranges = [g["range"] for g in got]
    assert ranges[0][0] == 0 and ranges[-1][1] == 160
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    assert all(r[0] % 32 == 0 for r in ranges)
    assert [g["slab_rows"] for g in got] == [-(-(r[1] - r[0]) // 16) for r in ranges]
