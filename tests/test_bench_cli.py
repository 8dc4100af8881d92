"""bench.py host logic without a GPU: the FLOP counts it reports, the
workload names, and the argument checks that run before any CUDA work."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ag_inputs  # noqa: E402
import bench  # noqa: E402


def test_forward_flops_count_two_products():
    w = ag_inputs.WORKLOADS["full"]
    # Q K^T and P V: 2 * L^2 * D multiply-adds each per (item, head).
    assert w.attn_flops() == 2 * (2 * 8 * 8192 * 8192 * 128)
    assert round(w.attn_flops() / 1e9, 1) == 274.9


def test_backward_flops_count_five_products():
    w = ag_inputs.WORKLOADS["full"]
    per_pair = {"S = Q K^T": 2 * 128, "dP = dO V^T": 2 * 128, "dV = P^T dO": 2 * 128,
                "dQ = dS K": 2 * 128, "dK = dS^T Q": 2 * 128}
    pairs = 1 * 8 * 8192 * 8192
    assert bench.backward_flops(w) == pairs * sum(per_pair.values())
    # Value width 128, tensor cores: S and dP in three passes (delta, keys,
    # dq), dout, P and dS each as two bf16 halves: pass 1 S + 2 dP, the key
    # pass S + 2 dP + 3 dV + 2 dK, pass 2 S + 2 dP + 2 dQ.
    executed = (1 + 2) + (1 + 2 + 3 + 2) + (1 + 2 + 2)
    assert bench.backward_executed_flops(w) == pairs * 2 * 128 * executed
    # Value width 192, CUDA cores: S and dP recomputed in three passes, the
    # three gradient products once each.
    w192 = ag_inputs.Workload("w192", B=1, L=8192, seed=0, Dv=192)
    executed = 3 * (2 * 128 + 2 * 192) + 2 * 128 + 2 * 128 + 2 * 192
    assert bench.backward_executed_flops(w192) == pairs * executed


def test_workload_names_follow_the_bias_mode():
    full = bench.workload_config(ag_inputs.WORKLOADS["full"])
    short = bench.workload_config(ag_inputs.WORKLOADS["short"])
    assert full["workload"] == "full_context_L8192_B1_projected_pair_bias"
    assert short["workload"] == "short_L2048_B1_direct_bias"


@pytest.mark.parametrize("argv,message", [
    (["--path", "backward", "--gpus", "2"], "one GPU"),
    (["--path", "backward", "--impl", "reference"], "one GPU"),
    (["--workload", "short"], "--path backward only"),
    (["--warmup", "2"], "at least 3"),
])
def test_bad_arguments_are_refused_before_any_work(argv, message):
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + argv,
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 2
    assert message in res.stderr
