#!/usr/bin/env python
"""Benchmark of the pair-bias multi-query attention hot path on B200.

One step = the whole path on one batch: ag_pair_bias_project (pair [512,512,128]
-> bias [8,512,512]) followed by ag_attn_fwd at full context (L = 8192, B = 1,
8 query heads sharing one K/V head, D = 128, 16x16 bias cells, cap 5).
The metric counts the attention's 4*B*H*L^2*D tensor FLOPs per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config tiny|short|mid|full|nine_block|all]

--config picks another of the workloads (default full, the headline line):
tiny/short/mid are L = 512/2048/4096 with a directly drawn bias, nine_block
runs nine independent L = 8192, B = 2 layers per step (each with its own
projected bias and cap); "all" prints one line per workload.
N > 1 runs under torchrun, one process per GPU; each rank runs its own
independent problem (weak scaling, no collective on the data path) and rank 0
prints one JSON line with the time taken as the maximum over ranks.
--impl reference times the float64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import ag_inputs  # noqa: E402

METRIC = "fused pair-bias attention TFLOP/s at L=8192, % of B200 BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = ag_inputs.WORKLOADS["full"]
FALLBACK_PEAK_TFLOPS = 1590.0
FLUSH_BYTES = 256 << 20
L2_NOTE = ("flushed between timed steps: a 256 MiB write, then a 256 MiB read so that "
           "the flush's own write-back of dirty lines happens before the timed region")


class L2Flush:
    """Evicts L2 between timed steps: writes a buffer larger than L2, then
    reads another one, so the next timed kernel finds a clean L2 instead of
    paying for the write-back of the flush's dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()
KERNEL_SOURCES = ["long_context_genomics_b200/csrc/attn_fwd_sm100.cu",
                  "long_context_genomics_b200/csrc/sm100.cuh"]


CONFIGS = ("tiny", "short", "mid", "full", "nine_block")


def workload_config(w) -> dict:
    return {
        "workload": (f"full_context_L{w.L}_B{w.B}_projected_pair_bias"
                     if w.bias_mode == "pair" else f"{w.name}_L{w.L}_B{w.B}_direct_bias"),
        "B": w.B, "L": w.L, "H": w.H, "D": w.D, "Dv": w.Dv, "P": w.P, "Cp": w.Cp,
        "block": w.block, "cap": w.cap, "seed": w.seed,
        "step": ("ag_pair_bias_project + ag_attn_fwd" if w.bias_mode == "pair"
                 else "ag_attn_fwd"),
        "l2": L2_NOTE,
    }


def config_layers(name: str) -> list:
    """The layers one step of a workload runs, in order."""
    if name == "nine_block":
        return list(ag_inputs.nine_block_stack().layers)
    return [ag_inputs.WORKLOADS[name]]


def job_config(name: str, layers: list, world: int) -> dict:
    """The line's config: the workload and, for the stack, every layer's cap
    and seed.  Both arms print the same keys."""
    if len(layers) == 1:
        cfg = workload_config(layers[0])
    else:
        w = layers[0]
        cfg = {"workload": f"nine_block_stack_L{w.L}_B{w.B}_projected_pair_bias",
               "layers": len(layers), "B": w.B, "L": w.L, "H": w.H, "D": w.D,
               "Dv": w.Dv, "P": w.P, "Cp": w.Cp, "block": w.block,
               "caps": [l.cap for l in layers], "seeds": [l.seed for l in layers],
               "step": f"{len(layers)} x (ag_pair_bias_project + ag_attn_fwd)",
               "l2": L2_NOTE}
    cfg["parallelism"] = f"{world} independent replicas" if world > 1 else "single GPU"
    return cfg


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return {"bf16_tflops": float(m["bf16_tflops"]), "hbm_gbs": float(m["hbm_gbs"]),
                "bf16_tflops_sustained": float(m.get("bf16_tflops_sustained", 0.0)) or None,
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16_tflops": FALLBACK_PEAK_TFLOPS, "hbm_gbs": 6650.0,
                "bf16_tflops_sustained": None, "source": "fallback"}


def _code_only(text: str) -> str:
    """The source without its comments and blank lines: an edit of comments
    alone leaves the kernel, and so its counters, unchanged."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    want = kernel_source_hash()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        fields = {}
        with open(path) as f:
            for line in f:
                item = line.strip().lstrip("-* ").strip("`")
                if ":" in item and item.startswith(("traffic_bytes_per_launch",
                                                    "kernel_source_sha256")):
                    k, v = item.split(":", 1)
                    fields[k.strip(" `")] = v.strip(" `")
        if fields.get("kernel_source_sha256") == want and "traffic_bytes_per_launch" in fields:
            try:
                return float(fields["traffic_bytes_per_launch"])
            except ValueError:
                return None
    return None


# --------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", uuid],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, RuntimeError, AttributeError):
            self.proc = None

    def stop(self, t0: float, t1: float) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != 8:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05] or rows[-5:]
        if not inside:
            return None
        reasons = sorted({name for r in inside for name, v in zip(self.REASONS, r[3])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# --------------------------------------------------------------------------
def _oracle_bias(orc, w, inp):
    return orc.pair_bias_project(inp["pair"], inp["W"]) if w.bias_mode == "pair" else inp["bias"]


def cpu_baseline(layers, min_s: float = 2.0) -> dict:
    """The float64 oracle, as it stands, on the host cores: one full pass over
    the first layer of the workload (every query row against every key;
    repeated while it takes under min_s, so that tiny workloads still get a
    stable time).  The bias comes from the oracle's own projection (untimed)."""
    import oracle

    orc = oracle.default()
    cores = orc.threads(len(os.sched_getaffinity(0)))
    w = layers[0]
    inp = ag_inputs.make_inputs(w)
    bias = _oracle_bias(orc, w, inp)
    passes, t = 0, 0.0
    while t < min_s:
        t0 = time.perf_counter()
        orc.attn_fwd(inp["q"], inp["k"], inp["v"], bias, block=w.block, cap=w.cap)
        t += time.perf_counter() - t0
        passes += 1
    what = "layer 1 of 9" if len(layers) > 1 else "the workload"
    return {"value": passes * w.attn_flops() / t / 1e12, "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{passes} full pass(es) over {what} (B={w.B}, L={w.L}: every query "
                      f"row against every key), float64, {t:.1f} s; projection untimed"}


def run_reference(args, rank: int, world: int) -> None:
    """The oracle on the host cores: each step is a bounded row sample of the
    workload's layers (full key range), sized so the whole run takes about
    two and a half minutes."""
    if rank != 0:
        return
    import oracle

    layers = config_layers(args.config)
    orc = oracle.default()
    cores = orc.threads(len(os.sched_getaffinity(0)))
    inps = [ag_inputs.make_inputs(w) for w in layers]
    biases = [_oracle_bias(orc, w, inp) for w, inp in zip(layers, inps)]
    w0 = layers[0]
    flops_row = 2.0 * w0.L * (w0.D + w0.Dv)
    per_step_s = min(6.0, 150.0 / max(1, args.steps + args.warmup))
    rows = ag_inputs.sample_rows(w0.B, w0.H, w0.L, max(4 * cores, 16), seed=0).numpy()
    t = time.perf_counter()
    orc.attn_rows(inps[0]["q"], inps[0]["k"], inps[0]["v"], biases[0], rows, block=w0.block,
                  cap=w0.cap)
    n = int(max(len(rows), len(rows) * per_step_s / max(time.perf_counter() - t, 1e-6)))
    n = min(n, w0.B * w0.H * w0.L)
    times, count = [], 0
    for s in range(args.warmup + args.steps):
        li = s % len(layers)  # the stack's layers take turns
        w, inp = layers[li], inps[li]
        rows = ag_inputs.sample_rows(w.B, w.H, w.L, n, seed=100 + s).numpy()
        t = time.perf_counter()
        orc.attn_rows(inp["q"], inp["k"], inp["v"], biases[li], rows, block=w.block, cap=w.cap)
        if s >= args.warmup:
            times.append(time.perf_counter() - t)
            count += len(rows)
    total = sum(times)
    value = count * flops_row / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": job_config(args.config, layers, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} random query rows per step (full key range) of "
                                   f"the workload's layers, float64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# Multi-rank plumbing (one process per GPU, launched by torchrun).  The ranks
# share no data: each runs its own independent problem, so the only
# collectives are the timing reductions below.
def rank_workload(base, rank: int):
    """Rank r's problem: the same shapes with its own input seed."""
    return dataclasses.replace(base, seed=base.seed + 1000 * rank)


def max_over_ranks(seconds: float, device, world: int) -> float:
    """The slowest rank's time: every rank calls this with its own device
    time (a collective, so all ranks must call it in the same order)."""
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def query_shard(L: int, world: int, rank: int) -> tuple:
    """Rank r's query positions [q0, q1) when the L queries of a sequence are
    split between the ranks: contiguous ranges, each a multiple of 32
    positions (whole pairs of 16-position blocks) except the last, which
    takes the remainder."""
    unit = 32
    units = -(-L // unit)
    q0 = min(L, unit * (units * rank // world))
    q1 = min(L, unit * (units * (rank + 1) // world))
    return q0, q1


def gather_keys(shard: torch.Tensor, world: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """All of a sequence's keys (or values) from every rank's contiguous
    shard [B, L/world, D]: one all_gather, the shards placed in rank order
    along the sequence.  out, if given, is the [B, L, D] result."""
    B, Ls, D = shard.shape
    if out is None:
        out = torch.empty(B, world * Ls, D, dtype=shard.dtype, device=shard.device)
    if world == 1:
        out.copy_(shard)
        return out
    parts = [torch.empty_like(shard) for _ in range(world)]
    torch.distributed.all_gather(parts, shard.contiguous())
    for r, part in enumerate(parts):
        out[:, r * Ls:(r + 1) * Ls].copy_(part)
    return out


def bias_rows(bias: torch.Tensor, q0: int, q1: int, block: int = 16) -> torch.Tensor:
    """The bias rows of query positions [q0, q1) (q0 a multiple of block):
    rows q0/block .. ceil(q1/block) of the last-but-one axis, contiguous."""
    assert q0 % block == 0
    return bias[..., q0 // block:-(-q1 // block), :].contiguous()


def check_device(ag, device: int, where: str) -> None:
    """Fails with the device error word's code (wait site << 8 | kind) if a
    bounded wait in one of the kernels ran out."""
    code = ag.ag_device_error(device)
    if code:
        raise RuntimeError(f"{where}: device error word {code:#x} (site {code >> 8})")


def aggregate_rate(world: int, units_per_step: float, steps: int, seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank does the same work per step)."""
    return world * units_per_step * steps / seconds


def _e2e_inputs(w) -> tuple:
    """The per-layer host inputs an end-to-end step uploads."""
    return ("q", "k", "v", "pair", "W") if w.bias_mode == "pair" else ("q", "k", "v", "bias")


def _forward(ag, w, d, bias, out, lse):
    """One layer through the public API: the projection (pair mode) and the
    attention."""
    if w.bias_mode == "pair":
        ag.ag_pair_bias_project(d["pair"], d["W"], bias=bias)
    else:
        bias = d["bias"]
    ag.ag_attn_fwd(d["q"], d["k"], d["v"], bias, cap=w.cap, out=out, lse=lse)


def pipelined_e2e(ag, layers, pinned: list, dev, steps: int):
    """Runs `steps` steps (every layer once per step) through the public API
    with each layer's inputs uploaded from pinned host memory and its out and
    lse downloaded again, as a pipeline: uploads, compute and downloads go on
    three streams, so one layer's upload and the previous one's download
    overlap the kernels in between.  Two device buffer sets keep an upload
    from overwriting inputs that a layer still reads and a layer from
    overwriting outputs that a download still reads.
    Returns (seconds from the first upload to the last download, the last
    layer's host lse)."""
    s_up, s_comp, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    w0 = layers[0]
    names = _e2e_inputs(w0)
    din = [{n: torch.empty(pinned[0][n].shape, dtype=pinned[0][n].dtype, device=dev)
            for n in names} for _ in range(2)]
    bias = torch.empty(w0.H, w0.P, w0.P, device=dev)   # produced and read on s_comp only
    dout = [torch.empty(w0.B, w0.H, w0.L, w0.Dv, device=dev) for _ in range(2)]
    dlse = [torch.empty(w0.B, w0.H, w0.L, device=dev) for _ in range(2)]
    hout = [torch.empty(dout[0].shape, pin_memory=True) for _ in range(2)]
    hlse = [torch.empty(dlse[0].shape, pin_memory=True) for _ in range(2)]
    in_ready, in_free, out_ready, out_free = (
        [torch.cuda.Event() for _ in range(2)] for _ in range(4))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(s_up)
    n = 0
    for _ in range(steps):
        for li, w in enumerate(layers):
            u = n % 2
            n += 1
            # A wait on an event not yet recorded (the first two) is a no-op.
            s_up.wait_event(in_free[u])          # the layer two back has read din[u]
            with torch.cuda.stream(s_up):
                for name in names:
                    din[u][name].copy_(pinned[li][name], non_blocking=True)
            in_ready[u].record(s_up)
            s_comp.wait_event(in_ready[u])
            s_comp.wait_event(out_free[u])       # its outputs are on the host
            with torch.cuda.stream(s_comp):
                _forward(ag, w, din[u], bias, dout[u], dlse[u])
            in_free[u].record(s_comp)
            out_ready[u].record(s_comp)
            s_down.wait_event(out_ready[u])
            with torch.cuda.stream(s_down):
                hout[u].copy_(dout[u], non_blocking=True)
                hlse[u].copy_(dlse[u], non_blocking=True)
            out_free[u].record(s_down)
    # The last download waits on every earlier stage, so t1 closes the run.
    t1.record(s_down)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / 1e3, hlse[(n - 1) % 2]


def run_ours(args, rank: int, world: int, local_rank: int) -> None:
    import long_context_genomics_b200 as ag

    dist = torch.distributed
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # Each rank runs its own independent problem (own seeds).
    layers = [rank_workload(w, rank) for w in config_layers(args.config)]
    hosts = [ag_inputs.make_inputs(w) for w in layers]
    pinned = [{n: t.pin_memory() for n, t in h.items()} for h in hosts]
    d = [{n: t.to(dev) for n, t in h.items()} for h in hosts]
    w0 = layers[0]
    biases = [torch.empty(w.H, w.P, w.P, device=dev) if w.bias_mode == "pair" else x["bias"]
              for w, x in zip(layers, d)]
    out = torch.empty(w0.B, w0.H, w0.L, w0.Dv, device=dev)
    lse = torch.empty(w0.B, w0.H, w0.L, device=dev)
    out_h = torch.empty(out.shape, pin_memory=True)
    lse_h = torch.empty(lse.shape, pin_memory=True)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    pair_mode = w0.bias_mode == "pair"

    def step():
        for w, x, b in zip(layers, d, biases):
            _forward(ag, w, x, b, out, lse)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    check_device(ag, local_rank, "after warm-up or timing")

    # ---- device-resident timing --------------------------------------------
    # Events per step: start, then after each layer's projection and after
    # its attention.
    K = args.steps
    nl = len(layers)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(1 + 2 * nl)] for _ in range(K)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.3 if sampler else 0.0)
    barrier()
    t_wall0 = time.time()
    for i in range(K):
        flush()                      # untimed: outside the events
        ev[i][0].record(stream)
        for li, (w, x, b) in enumerate(zip(layers, d, biases)):
            if pair_mode:
                ag.ag_pair_bias_project(x["pair"], x["W"], bias=b)
            ev[i][1 + 2 * li].record(stream)
            ag.ag_attn_fwd(x["q"], x["k"], x["v"], b, cap=w.cap, out=out, lse=lse)
            ev[i][2 + 2 * li].record(stream)
    barrier()
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None
    step_ms = [e[0].elapsed_time(e[-1]) for e in ev]
    proj_ms = [sum((e[2 * li] if li else e[0]).elapsed_time(e[1 + 2 * li]) for li in range(nl))
               for e in ev]
    attn_ms = [sum(e[1 + 2 * li].elapsed_time(e[2 + 2 * li]) for li in range(nl)) for e in ev]
    total_s = max_over_ranks(sum(step_ms) / 1e3, dev, world)
    check_device(ag, local_rank, "after warm-up or timing")

    # ---- end to end through the public API with host buffers ---------------
    names = _e2e_inputs(w0)
    h2d = sum(pinned[li][n].numel() * pinned[li][n].element_size()
              for li in range(nl) for n in names)
    d2h = nl * (out_h.numel() * 4 + lse_h.numel() * 4)
    # (1) Pipelined, as a serving loop runs it: every step's copies are inside
    # the timed region, overlapped with the neighbouring layers' kernels.
    pipelined_e2e(ag, layers, pinned, dev, max(1, min(args.warmup, 3)))
    barrier()
    e2e_s, e2e_lse = pipelined_e2e(ag, layers, pinned, dev, K)
    e2e_s = max_over_ranks(e2e_s, dev, world)
    check_device(ag, local_rank, "e2e pipelined")
    assert math.isfinite(float(e2e_lse.flatten()[0]))
    # (2) One layer at a time on one stream: upload, compute, download.
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier()
    for i in range(K):
        flush()
        ee[i][0].record(stream)
        for li, (w, x, b) in enumerate(zip(layers, d, biases)):
            for n in names:
                x[n].copy_(pinned[li][n], non_blocking=True)
            _forward(ag, w, x, b, out, lse)
            out_h.copy_(out, non_blocking=True)
            lse_h.copy_(lse, non_blocking=True)
        ee[i][1].record(stream)
    barrier()
    serial_s = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ee) / 1e3, dev, world)
    check_device(ag, local_rank, "e2e serial")
    assert math.isfinite(float(lse_h.flatten()[0]))

    if rank != 0:
        return
    flops = sum(w.attn_flops() for w in layers)
    attn_bytes = sum(w.attn_bytes() for w in layers)
    proj_bytes = sum(w.project_bytes() for w in layers) if pair_mode else 0
    pk = peaks()
    value = aggregate_rate(world, flops, K, total_s) / 1e12
    attn_mean_s = statistics.mean(attn_ms) / 1e3
    attn_med_s = statistics.median(attn_ms) / 1e3
    achieved = flops / attn_mean_s / 1e12
    launches = sum(ag.ag_attn_fwd_launch_count(w.B, w.L, w.cap) for w in layers)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": job_config(args.config, layers, world),
        "pct_of_peak": 100.0 * (value / world) / pk["bf16_tflops"],
        "peak_source": pk["source"],
        "e2e": {"value": aggregate_rate(world, flops, K, e2e_s) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": 1e3 * e2e_s / K,
                "schedule": "pipelined: uploads, compute and downloads on three "
                            "streams, two device buffer sets",
                "l2": f"inputs uploaded every step ({h2d / 1e6:.0f} MB); no flush"},
        "e2e_serial": {"value": aggregate_rate(world, flops, K, serial_s) / 1e12,
                       "unit": UNIT, "ms_per_step": 1e3 * serial_s / K,
                       "schedule": "one stream: upload, compute, download per layer"},
        # Our kernels in the timed region: per layer the projection (pair
        # mode) and the attention's one or two launches.
        "gpu_launches": K * ((nl if pair_mode else 0) + launches),
        "roofline": {"kernel": "attn_fwd_kernel", "bound": "tensor", "achieved": achieved,
                     "peak": pk["bf16_tflops"], "unit": UNIT,
                     "frac": achieved / pk["bf16_tflops"], "traffic": profiled_traffic(),
                     "peak_kind": "bf16 burst (" + pk["source"] + ")",
                     # Context: the same rate against the power-capped figure
                     # (a GEMM looped for seconds at the 1 kW limit).
                     "frac_of_sustained": (achieved / pk["bf16_tflops_sustained"]
                                           if pk["bf16_tflops_sustained"] else None)},
        "attn_ms": {"median": 1e3 * attn_med_s,
                    "p95": sorted(attn_ms)[int(0.95 * (K - 1))],
                    "tflops_median": flops / attn_med_s / 1e12,
                    "pct_of_peak_median": 100.0 * flops / attn_med_s / 1e12 / pk["bf16_tflops"],
                    "algorithmic_gbs": attn_bytes / attn_med_s / 1e9},
        "clocks": clocks,
    }
    if pair_mode:
        proj_mean_s = statistics.mean(proj_ms) / 1e3
        line["projection"] = {"ms_median": statistics.median(proj_ms),
                              "achieved_gbs": proj_bytes / proj_mean_s / 1e9,
                              "peak_gbs": pk["hbm_gbs"],
                              "frac": proj_bytes / proj_mean_s / 1e9 / pk["hbm_gbs"]}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(layers)
    print(json.dumps(line), flush=True)


def run_sharded(args, rank: int, world: int, local_rank: int) -> None:
    """One full-context problem split between the ranks by query position
    (strong scaling).  Each rank holds its slab of queries, its rows of the
    pair representation and a contiguous shard of the keys and values, as a
    sequence-parallel model would; every step all-gathers K and V (NCCL),
    projects its pair rows and runs the attention for its queries.  The
    outputs stay sharded: no collective follows."""
    import long_context_genomics_b200 as ag

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = config_layers(args.config)[0]
    if len(config_layers(args.config)) != 1 or w.bias_mode != "pair":
        raise SystemExit("--shard queries runs the single-layer projected workload (full)")
    host = ag_inputs.make_inputs(w)       # every rank draws the same problem
    q0, q1 = query_shard(w.L, world, rank)
    k0, k1 = w.L * rank // world, w.L * (rank + 1) // world
    if (w.L % world) or (w.L // world) % 16:
        raise SystemExit("--shard queries needs L / world to be a multiple of 16")
    q = host["q"][:, :, q0:q1].contiguous().to(dev)
    k_shard = host["k"][:, k0:k1].contiguous().to(dev)
    v_shard = host["v"][:, k0:k1].contiguous().to(dev)
    pair = host["pair"][q0 // 16:-(-q1 // 16)].contiguous().to(dev)   # pair rows of the slab
    W = host["W"].to(dev)
    k_full = torch.empty(w.B, w.L, w.D, dtype=torch.bfloat16, device=dev)
    v_full = torch.empty(w.B, w.L, w.Dv, dtype=torch.bfloat16, device=dev)
    bias = torch.empty(w.H, pair.shape[0], w.P, device=dev)
    out = torch.empty(w.B, w.H, q1 - q0, w.Dv, device=dev)
    lse = torch.empty(w.B, w.H, q1 - q0, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step():
        gather_keys(k_shard, world, k_full)
        gather_keys(v_shard, world, v_full)
        ag.ag_pair_bias_project_rows(pair, W, bias=bias)
        ag.ag_attn_fwd_query_slab(q, k_full, v_full, bias, cap=w.cap, out=out, lse=lse)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush()
        step()
    barrier()
    check_device(ag, local_rank, "after warm-up or timing")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.3 if sampler else 0.0)
    barrier()
    t_wall0 = time.time()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    barrier()
    clocks = sampler.stop(t_wall0, time.time()) if sampler else None
    total_s = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3, dev, world)
    check_device(ag, local_rank, "sharded timing")
    assert math.isfinite(float(lse[0, 0, 0]))
    if rank != 0:
        return
    pk = peaks()
    flops = w.attn_flops()                # the whole problem, split between the ranks
    value = flops * K / total_s / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": 1e3 * total_s / K, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**job_config(args.config, [w], 1),
                   "parallelism": f"queries split over {world} GPUs (K/V all-gather)",
                   "step": "all_gather K, V + ag_pair_bias_project_rows + "
                           "ag_attn_fwd_query_slab"},
        "pct_of_peak": 100.0 * value / world / pk["bf16_tflops"], "peak_source": pk["source"],
        "gpu_launches": K * (1 + 2), "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def backward_flops(w) -> float:
    """Algorithmic FLOPs of one backward call, the usual count of five L x L
    products: S = Q K^T (recomputed), dP = dO V^T, dV = P^T dO, dQ = dS K,
    dK = dS^T Q, i.e. 2 B H L^2 (3 D + 2 Dv)."""
    return 2.0 * w.B * w.H * w.L * w.L * (3 * w.D + 2 * w.Dv)


def backward_executed_flops(w) -> float:
    """FLOPs the backward kernels execute per call.  Value width 128 (tensor
    cores, dout, P and dS each taken as a pair of bf16 halves): query pass 1
    S + 2 dP, the key pass S^T + 2 dP^T + 3 dV + 2 dK, query pass 2
    S + 2 dP + 2 dQ, i.e. 16 products of 2 L^2 x 128 per (item, head).
    Value width 192 (CUDA cores): the delta pass 2 (D + Dv), the dq pass
    2 (D + Dv) + 2 D and the key kernel 2 (D + Dv) + 2 D + 2 Dv per
    (item, head, query, key)."""
    if w.Dv == 128:
        return 2.0 * w.B * w.H * w.L * w.L * 128 * 16
    return 2.0 * w.B * w.H * w.L * w.L * (3 * (w.D + w.Dv) + 2 * w.D + w.Dv)


def run_backward(args) -> None:
    """One GPU: ag_attn_bwd on one workload (by default the full-context one
    with its projected bias), given the forward's lse, timed per call with
    CUDA events, L2 flushed between calls."""
    import long_context_genomics_b200 as ag

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = ag_inputs.WORKLOADS[args.workload]
    host = ag_inputs.make_inputs(w)
    d = {n: t.to(dev) for n, t in host.items()}
    bias = ag.ag_pair_bias_project(d["pair"], d["W"]) if "pair" in d else d["bias"]
    _, lse = ag.ag_attn_fwd(d["q"], d["k"], d["v"], bias, cap=w.cap)
    g = torch.Generator(device="cpu").manual_seed(w.seed + 500)
    dout = torch.randn(w.B, w.H, w.L, w.Dv, generator=g).to(dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush()
        ag.ag_attn_bwd(d["q"], d["k"], d["v"], bias, lse, dout, cap=w.cap)
    torch.cuda.synchronize()
    check_device(ag, 0, "backward")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(0)
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        ag.ag_attn_bwd(d["q"], d["k"], d["v"], bias, lse, dout, cap=w.cap)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop(t0, time.time())
    check_device(ag, 0, "backward")
    ms = [e[0].elapsed_time(e[1]) for e in ev]
    mean_s = statistics.mean(ms) / 1e3
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    max_mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    alg = backward_flops(w) / mean_s / 1e12
    exe = backward_executed_flops(w) / mean_s / 1e12
    if w.Dv == 128:
        pk = peaks()
        roof = {"kernel": "bwd_query_kernel x 2 + bwd_key_kernel (tcgen05)", "bound": "tensor",
                "achieved": alg, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": alg / pk["bf16_tflops"], "traffic": None,
                "peak_kind": "bf16 burst (" + pk["source"] + ")",
                "executed_tflops": exe, "frac_executed": exe / pk["bf16_tflops"]}
        dtype = "bf16"
    else:
        # FP32 FMA pipe: 128 lanes per SM, 2 FLOPs per FMA, at the maximum SM clock.
        fp32_peak = sms * 128 * 2 * max_mhz * 1e6 / 1e12
        roof = {"kernel": "attn_bwd_q_kernel + attn_bwd_kv_kernel", "bound": "alu",
                "achieved": alg, "peak": fp32_peak, "unit": "TFLOP/s",
                "frac": alg / fp32_peak, "traffic": None,
                "peak_kind": f"fp32 FMA pipe, {sms} SMs x 128 lanes x 2 x {max_mhz:.0f} MHz",
                "executed_tflops": exe, "frac_executed": exe / fp32_peak}
        dtype = "f32"
    line = {
        "metric": f"pair-bias attention backward TFLOP/s at L={w.L}", "value": alg,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": 1e3 * mean_s, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {**workload_config(w), "step": "ag_attn_bwd (given the forward's lse)",
                   "parallelism": "single GPU"},
        "gpu_launches": K * ag.ag_attn_bwd_launch_count(w.Dv),
        "roofline": roof,
        "ms": {"median": statistics.median(ms), "p95": sorted(ms)[int(0.95 * (K - 1))]},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; 20 with --path backward)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--path", choices=["forward", "backward"], default="forward",
                    help="forward: projection + attention (the default step); "
                         "backward: the attention backward alone, one GPU")
    ap.add_argument("--workload", choices=sorted(ag_inputs.WORKLOADS), default="full",
                    help="with --path backward: which workload (default full, L=8192)")
    ap.add_argument("--config", choices=CONFIGS + ("all",), default="full",
                    help="forward workload (default full: L=8192, B=1, the headline line)")
    ap.add_argument("--shard", choices=["replicas", "queries"], default="replicas",
                    help="N > 1: independent problems per GPU (replicas, weak scaling) or "
                         "one problem's queries split between the GPUs (strong scaling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 20 if args.path == "backward" else 1000
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.path == "backward":
        if args.gpus != 1 or args.impl != "ours":
            ap.error("--path backward runs our kernels on one GPU")
    elif args.workload != "full":
        ap.error("--workload applies to --path backward only")
    if args.path == "backward" and args.config != "full":
        ap.error("--config applies to --path forward")
    if args.shard == "queries" and (args.config != "full" or args.impl != "ours"):
        ap.error("--shard queries runs our kernels on the full workload")
    if args.path == "backward":
        run_backward(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            sys.exit("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    configs = CONFIGS if args.config == "all" else (args.config,)
    if args.impl == "reference":
        # Rank 0 alone times the oracle; the other ranks exit without work.
        for c in configs:
            run_reference(argparse.Namespace(**{**vars(args), "config": c}), rank, world)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(
            backend="nccl", timeout=datetime.timedelta(seconds=120))
    try:
        for c in configs:
            a = argparse.Namespace(**{**vars(args), "config": c})
            if args.shard == "queries":
                run_sharded(a, rank, world, local_rank)
            else:
                run_ours(a, rank, world, local_rank)
            torch.cuda.empty_cache()
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
