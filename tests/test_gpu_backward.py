"""Backward kernels against the float64 oracle on B200 (CUDA path through the
C ABI).  The forward kernel supplies lse, as a training step would.

Tolerance, per gradient tensor: max |gpu - oracle| <= 3e-3 * max |oracle|.
Two things separate the kernels from the oracle.  (1) lse comes from the
forward kernel, whose own bound is 1e-3; an error e in lse_i scales every
p_ij of the row, and through delta_i every ds_ij, by exp(-e), so a gradient
moves by about 2e relative to the size of its terms.  (2) The kernels sum
up to L = 8192 fp32 terms per value: at most L * 2^-24 = 4.9e-4 relative.
Both together stay under 2.5e-3; 3e-3 is the bound.
"""
import math

import numpy as np
import pytest
import torch

import ag_inputs

pytestmark = pytest.mark.gpu

TOL = 3e-3


@pytest.fixture(scope="module")
def ag():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_genomics_b200 as ag

    return ag


def _run(ag, c, dout, cap):
    dev = "cuda"
    q, k, v, bias = (c[n].to(dev) for n in ("q", "k", "v", "bias"))
    out, lse = ag.ag_attn_fwd(q, k, v, bias, cap=cap)
    grads = ag.ag_attn_bwd(q, k, v, bias, lse, dout.to(dev), cap=cap)
    torch.cuda.synchronize()
    assert ag.ag_device_error(0) == 0
    return [g.cpu().double().numpy() for g in grads], out.cpu().double().numpy()


def _dout(B, L, Dv, seed):
    return torch.randn(B, 8, L, Dv, generator=torch.Generator().manual_seed(seed))


def _close(name, got, want):
    scale = float(np.abs(want).max())
    err = float(np.abs(got - want).max())
    assert err <= TOL * scale, f"{name}: max |diff| {err:.3e} > {TOL} * {scale:.3e}"


@pytest.mark.parametrize("B,L,Dv,cap,batched", [
    (1, 256, 128, 5.0, False),
    (2, 200, 128, 5.0, False),      # partial last block; one bias for both items
    (2, 136, 192, math.inf, True),  # value width 192, no cap, one bias per item
    (1, 33, 128, 30.0, False),
    (3, 64, 128, 5.0, True),
    (2, 16, 128, 5.0, False),       # one query block: one CTA of the key pair has none
    (1, 1000, 128, 40.0, False),    # many steps per tile and per key CTA, ragged end
    (160, 128, 128, 5.0, False),    # many items: accumulators restarted many times per CTA
    (48, 250, 128, math.inf, True), # many ragged items, one bias per item, no cap
])
def test_backward_parity(ag, oracle_lib, B, L, Dv, cap, batched):
    c = ag_inputs.random_case(B, 8, L, 128, Dv, 16, seed=L + B, batched_bias=batched)
    dout = _dout(B, L, Dv, seed=L)
    (dq, dk, dv, db, delta), _ = _run(ag, c, dout, cap)
    rq, rk, rv, rb, _, rd = oracle_lib.attn_bwd(c["q"], c["k"], c["v"], c["bias"], dout,
                                                block=16, cap=cap)
    for name, g, w in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv), ("dbias", db, rb),
                       ("delta", delta, rd)):
        _close(name, g, w)


def test_backward_full_context_sampled(ag, oracle_lib):
    """L = 8192, B = 1: sampled rows of dq, keys of dk and dv, and bias cells,
    including the first and last of each."""
    L = 8192
    c = ag_inputs.random_case(1, 8, L, 128, 128, 16, seed=3)
    dout = _dout(1, L, 128, seed=4)
    (dq, dk, dv, db, _), _ = _run(ag, c, dout, 5.0)
    rng = np.random.default_rng(5)
    rows = [[0, 0, 0], [0, 7, L - 1]] + [[0, int(h), int(i)] for h, i in
                                        zip(rng.integers(0, 8, 10), rng.integers(0, L, 10))]
    keys = [[0, 0], [0, L - 1]] + [[0, int(j)] for j in rng.integers(0, L, 10)]
    P = L // 16
    cells = [[0, 0, 0, 0], [0, 7, P - 1, P - 1]] + [
        [0, int(h), int(I), int(J)] for h, I, J in
        zip(rng.integers(0, 8, 10), rng.integers(0, P, 10), rng.integers(0, P, 10))]
    sq, sk, sv, sb = oracle_lib.attn_bwd_sample(c["q"], c["k"], c["v"], c["bias"], dout,
                                                rows=rows, keys=keys, cells=cells,
                                                block=16, cap=5.0)
    _close("dq rows", np.stack([dq[b, h, i] for b, h, i in rows]), sq)
    _close("dk keys", np.stack([dk[b, j] for b, j in keys]), sk)
    _close("dv keys", np.stack([dv[b, j] for b, j in keys]), sv)
    _close("dbias cells", np.array([db[h, I, J] for _, h, I, J in cells]), sb)


def test_backward_delta_matches_the_forward_output(ag):
    """delta_i = sum_j p_ij (dout_i . v_j) equals dout_i . out_i, with out
    from the forward kernel (whose own error bounds the difference)."""
    c = ag_inputs.random_case(1, 8, 512, 128, 128, 16, seed=9)
    dout = _dout(1, 512, 128, seed=10)
    (_, _, _, _, delta), out = _run(ag, c, dout, 5.0)
    want = np.einsum("bhic,bhic->bhi", dout.double().numpy(), out)
    assert float(np.abs(delta - want).max()) <= 2e-2 * float(dout.abs().sum(-1).max())


def test_backward_is_deterministic(ag):
    c = ag_inputs.random_case(2, 8, 160, 128, 128, 16, seed=11)
    dout = _dout(2, 160, 128, seed=12)
    a, _ = _run(ag, c, dout, 5.0)
    b, _ = _run(ag, c, dout, 5.0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_empty_is_a_noop(ag):
    z = torch.zeros(0, 8, 64, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(0, 64, 128, dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(8, 4, 4, device="cuda")
    lse = torch.zeros(0, 8, 64, device="cuda")
    dout = torch.zeros(0, 8, 64, 128, device="cuda")
    dq, dk, dv, db, delta = ag.ag_attn_bwd(z, kv, kv, bias, lse, dout)
    assert dq.shape == (0, 8, 64, 128) and dk.shape == (0, 64, 128) and db.shape == (8, 4, 4)
