"""GPU parity: libag's kernels against the float64 oracle on the same seeded
inputs (bf16 q/k/v and fp32 bias widened exactly).

Tolerances (bf16 inputs, fp32 accumulation): max |out - oracle| <= 2e-2 and
max |lse - oracle| <= 1e-3; projection: fp32 sums of 128 products,
max |bias - oracle| <= 1e-4.
"""
import math

import numpy as np
import pytest
import torch

import ag_inputs

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
LSE_TOL = 1e-3
PROJ_TOL = 1e-4


@pytest.fixture(scope="module")
def ag():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_genomics_b200 as ag

    return ag


def _dev(t):
    return t.to("cuda").contiguous()


def _gpu_attn(ag, inp, cap, bias=None, stream=None):
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    b = _dev(inp["bias"]) if bias is None else bias
    out, lse = ag.ag_attn_fwd(q, k, v, b, cap=cap, stream=stream)
    torch.cuda.synchronize()
    assert ag.ag_device_error(0) == 0
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def _compare(out, lse, ref_out, ref_lse, what):
    assert np.isfinite(out).all() and np.isfinite(lse).all(), f"{what}: non-finite"
    eo = float(np.max(np.abs(out - ref_out))) if out.size else 0.0
    el = float(np.max(np.abs(lse - ref_lse))) if lse.size else 0.0
    print(f"{what}: max|dout|={eo:.3e} max|dlse|={el:.3e}")
    assert eo <= OUT_TOL, f"{what}: max|dout| {eo:.3e} > {OUT_TOL}"
    assert el <= LSE_TOL, f"{what}: max|dlse| {el:.3e} > {LSE_TOL}"
    return eo, el


# --------------------------------------------------------------------------
@pytest.mark.parametrize("P", [1, 3, 5, 32, 128, 512])
def test_projection_parity(ag, oracle_lib, P):
    g = torch.Generator().manual_seed(100 + P)
    pair = torch.randn(P, P, 128, generator=g)
    W = torch.randn(128, 8, generator=g) / math.sqrt(128)
    bias = ag.ag_pair_bias_project(_dev(pair), _dev(W))
    torch.cuda.synchronize()
    ref = oracle_lib.pair_bias_project(pair, W)
    err = float(np.max(np.abs(bias.double().cpu().numpy() - ref)))
    print(f"projection P={P}: max|d|={err:.3e}")
    assert err <= PROJ_TOL


@pytest.mark.parametrize("name", ["tiny", "short", "mid"])
def test_config_parity_full(ag, oracle_lib, name):
    w = ag_inputs.WORKLOADS[name]
    inp = ag_inputs.make_inputs(w)
    out, lse = _gpu_attn(ag, inp, w.cap)
    ref_out, ref_lse = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                           block=16, cap=w.cap)
    eo, _ = _compare(out, lse, ref_out, ref_lse, name)
    if name == "tiny":
        # For context: the page's standalone L=512 tiled-vs-dense figure was
        # 2^-9 max abs error (a different pair of bf16 paths, not a bound).
        print(f"tiny max|dout| {eo:.3e} vs page figure 1.953e-03")


def test_full_context_with_projection_sampled(ag, oracle_lib):
    """L = 8192 with the projected pair bias, exactly as the benchmark runs it;
    2048 sampled rows against the oracle, every row checked for finiteness."""
    w = ag_inputs.WORKLOADS["full"]
    inp = ag_inputs.make_inputs(w)
    bias = ag.ag_pair_bias_project(_dev(inp["pair"]), _dev(inp["W"]))
    out, lse = _gpu_attn(ag, inp, w.cap, bias=bias)
    ref_bias = oracle_lib.pair_bias_project(inp["pair"], inp["W"])
    assert float(np.max(np.abs(bias.double().cpu().numpy() - ref_bias))) <= PROJ_TOL
    rows = ag_inputs.sample_rows(w.B, w.H, w.L, 2048, seed=7).numpy()
    # The oracle uses its own projected bias: the two paths share nothing.
    ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], ref_bias, rows,
                                  block=16, cap=w.cap)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    _compare(out[b, h, i], lse[b, h, i], ro, rl, "full L=8192 sampled")
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    assert (lse <= w.cap + math.log(w.L) + 1e-3).all()


def test_nine_block_stack_sampled(ag, oracle_lib):
    for layer in ag_inputs.nine_block_stack().layers:
        inp = ag_inputs.make_inputs(layer)
        bias = ag.ag_pair_bias_project(_dev(inp["pair"]), _dev(inp["W"]))
        out, lse = _gpu_attn(ag, inp, layer.cap, bias=bias)
        ref_bias = oracle_lib.pair_bias_project(inp["pair"], inp["W"])
        rows = ag_inputs.sample_rows(layer.B, layer.H, layer.L, 192,
                                     seed=layer.seed).numpy()
        ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], ref_bias, rows,
                                      block=16, cap=layer.cap)
        b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
        _compare(out[b, h, i], lse[b, h, i], ro, rl,
                 f"{layer.name} cap={layer.cap}")


@pytest.mark.parametrize("B,L", [(1, 16), (2, 48), (1, 128), (1, 144), (3, 400),
                                 (1, 1040), (2, 2064)])
@pytest.mark.parametrize("cap", [5.0, math.inf])
def test_ragged_and_odd_shapes(ag, oracle_lib, B, L, cap):
    """L not a multiple of the 128-key tile (masked tail) and odd numbers of
    16-position blocks (the last pair of a batch item has one tile)."""
    inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=B * 1000 + L)
    out, lse = _gpu_attn(ag, inp, cap)
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=cap)
    _compare(out, lse, ro, rl, f"B={B} L={L} cap={cap}")


@pytest.mark.parametrize("B,L", [(160, 128), (48, 250)])
@pytest.mark.parametrize("cap", [5.0, 50.0, math.inf])
def test_many_short_segments_per_cluster(ag, oracle_lib, B, L, cap):
    """Many items of one or two key tiles: every cluster runs several short
    segments in a row, so the output accumulator is read out and restarted
    many times per launch, and with one-tile segments each softmax group
    owns every other segment's only tile."""
    inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=B * 1000 + L + 7)
    out, lse = _gpu_attn(ag, inp, cap)
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=cap)
    _compare(out, lse, ro, rl, f"B={B} L={L} cap={cap}")


@pytest.mark.parametrize("B,L", [(1, 1), (1, 17), (2, 100), (1, 1000), (3, 2049),
                                 (1, 4095)])
@pytest.mark.parametrize("cap", [5.0, 50.0, math.inf])
def test_lengths_with_a_partial_block(ag, oracle_lib, B, L, cap):
    """L not a multiple of 16: the last query block and the last bias cell
    cover fewer than 16 positions (P = ceil(L/16)); rows past L are never
    written."""
    inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=B * 7919 + L)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    bias = _dev(inp["bias"])
    out = torch.full((B, 8, L, 128), float("nan"), device="cuda")
    lse = torch.full((B, 8, L), float("nan"), device="cuda")
    ag.ag_attn_fwd(q, k, v, bias, cap=cap, out=out, lse=lse)
    torch.cuda.synchronize()
    assert ag.ag_device_error(0) == 0
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=cap)
    _compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl,
             f"B={B} L={L} cap={cap}")


@pytest.mark.parametrize("B,L", [(3, 1040), (2, 333), (2, 8192)])
@pytest.mark.parametrize("cap", [5.0, math.inf])
def test_one_bias_per_batch_item(ag, oracle_lib, B, L, cap):
    """bias [B,H,P,P] (ag_attn_fwd_strided_bias): each batch item reads its
    own bias; full outputs against the oracle (sampled rows at L = 8192)."""
    inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=B * 31 + L,
                                batched_bias=True)
    out, lse = _gpu_attn(ag, inp, cap)
    if L <= 2048:
        ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                     block=16, cap=cap)
        _compare(out, lse, ro, rl, f"per-item bias B={B} L={L} cap={cap}")
    else:
        rows = ag_inputs.sample_rows(B, 8, L, 384, seed=L).numpy()
        ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], inp["bias"], rows,
                                      block=16, cap=cap)
        b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
        _compare(out[b, h, i], lse[b, h, i], ro, rl, f"per-item bias B={B} L={L} sampled")


@pytest.mark.parametrize("B,L", [(1, 512), (2, 1040), (1, 2049)])
@pytest.mark.parametrize("cap", [5.0, 50.0, math.inf])
def test_value_width_192(ag, oracle_lib, B, L, cap):
    """Dv = 192 (the page's checkpoint value width) through ag_attn_fwd_ex:
    v [B,L,192], out [B,H,L,192], scale still 1/sqrt(128)."""
    inp = ag_inputs.random_case(B, 8, L, 128, 192, 16, seed=B * 97 + L)
    out, lse = _gpu_attn(ag, inp, cap)
    assert out.shape == (B, 8, L, 192)
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=cap)
    _compare(out, lse, ro, rl, f"Dv=192 B={B} L={L} cap={cap}")


def test_value_width_192_full_context_sampled(ag, oracle_lib):
    """Dv = 192 at L = 8192 with one bias per batch item (B = 2): split pairs
    and the merge run; sampled rows against the oracle."""
    B, L = 2, 8192
    inp = ag_inputs.random_case(B, 8, L, 128, 192, 16, seed=192, batched_bias=True)
    out, lse = _gpu_attn(ag, inp, 5.0)
    rows = ag_inputs.sample_rows(B, 8, L, 512, seed=19).numpy()
    ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], inp["bias"], rows,
                                  block=16, cap=5.0)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    _compare(out[b, h, i], lse[b, h, i], ro, rl, "Dv=192 L=8192 sampled")
    assert np.isfinite(out).all() and np.isfinite(lse).all()


def test_strided_bias_with_padding_between_items(ag, oracle_lib):
    """A bias batch stride larger than H*P*P (padded items) through the C ABI."""
    import ctypes
    B, L = 2, 400
    P = 25
    inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=5, batched_bias=True)
    stride = 8 * P * P + 96
    padded = torch.full((B, stride), float("nan"))
    padded[:, : 8 * P * P] = inp["bias"].reshape(B, -1)
    q, k, v, bp = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(padded)
    out = torch.empty(B, 8, L, 128, device="cuda")
    lse = torch.empty(B, 8, L, device="cuda")
    st = ag.lib.ag_attn_fwd_strided_bias(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), bp.data_ptr(), stride, B, 8, L, 128,
        16, ctypes.c_float(5.0), out.data_ptr(), lse.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
    assert ag.ag_device_error(0) == 0
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"], block=16,
                                 cap=5.0)
    _compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl,
             "padded per-item bias")


@pytest.mark.parametrize("cap", [1.0, 5.0, 10.0, 30.0, 40.0, 50.0, 60.0, 61.0, 1e4, math.inf])
def test_cap_modes(ag, oracle_lib, cap):
    """Static shift (cap <= 60; shift ceil(cap log2 e) up to cap 41.6, then
    120 - that), running max with the cap (cap > 60) and no cap at all."""
    inp = ag_inputs.random_case(2, 8, 512, 128, 128, 16, seed=int(min(cap, 1e6)) + 3)
    out, lse = _gpu_attn(ag, inp, cap)
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=cap)
    _compare(out, lse, ro, rl, f"cap={cap}")


@pytest.mark.parametrize("cap", [5.0, 10.0, 30.0, 40.0, 50.0, 60.0, 61.0, math.inf])
def test_large_logits(ag, oracle_lib, cap):
    """q, k with std 3 and a bias of std 4: logits far beyond the cap
    (saturated tanh), a softmax dominated by a few keys at the large caps
    (where an error in a logit passes straight into lse) and, without a cap,
    a wide softmax range.  Caps 40 and 50 sit on either side of the switch
    between the two shifts of the static mode, 60 and 61 on either side of
    the switch to the running maximum."""
    inp = ag_inputs.random_case(1, 8, 640, 128, 128, 16, seed=77, bias_std=4.0,
                                qk_std=3.0)
    out, lse = _gpu_attn(ag, inp, cap)
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=cap)
    _compare(out, lse, ro, rl, f"large logits cap={cap}")


@pytest.mark.parametrize("cap", [5.0, 10.0, 40.0, 50.0, 60.0, 61.0])
def test_large_logits_full_context_sampled(ag, oracle_lib, cap):
    """The same logit distribution at L = 8192 (8192 keys per softmax, the
    two-launch schedule at B = 1), sampled rows against the oracle."""
    inp = ag_inputs.random_case(1, 8, 8192, 128, 128, 16, seed=78, bias_std=4.0,
                                qk_std=3.0)
    out, lse = _gpu_attn(ag, inp, cap)
    rows = ag_inputs.sample_rows(1, 8, 8192, 384, seed=int(cap)).numpy()
    ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], inp["bias"], rows,
                                  block=16, cap=cap)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    _compare(out[b, h, i], lse[b, h, i], ro, rl, f"large logits L=8192 cap={cap} sampled")


def test_split_pairs_full_context(ag, oracle_lib):
    """L = 8192, B = 1 on a 148-SM B200 runs two launches: the last 74 pairs
    of query blocks (positions 5824..8191) have their keys split in two, the
    second launch merging into the first's results.  Rows drawn from those
    positions only, all heads, against the oracle."""
    w = ag_inputs.WORKLOADS["full"]
    inp = ag_inputs.make_inputs(w)
    bias = ag.ag_pair_bias_project(_dev(inp["pair"]), _dev(inp["W"]))
    out, lse = _gpu_attn(ag, inp, w.cap, bias=bias)
    ref_bias = oracle_lib.pair_bias_project(inp["pair"], inp["W"])
    g = torch.Generator().manual_seed(8)
    pos = 5824 + torch.randperm(8192 - 5824, generator=g)[:64]
    rows = np.array([(0, h, int(i)) for i in pos for h in range(8)] +
                    [(0, h, i) for i in (5824, 5855, 5856, 8191) for h in range(8)])
    ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], ref_bias, rows,
                                  block=16, cap=w.cap)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    _compare(out[b, h, i], lse[b, h, i], ro, rl, "split pairs L=8192")


def test_two_streams_at_once(ag, oracle_lib):
    """Two different L = 8192 calls issued on two streams without waiting for
    each other (the library keeps no shared scratch, so they may overlap on
    the GPU): one B = 1 (two launches) and one B = 2 with its own bias per
    item (whole pairs), each checked against the oracle on sampled rows."""
    cases = [ag_inputs.random_case(1, 8, 8192, 128, 128, 16, seed=61),
             ag_inputs.random_case(2, 8, 8192, 128, 128, 16, seed=62, batched_bias=True)]
    dev = [{n: _dev(t) for n, t in c.items()} for c in cases]
    outs = []
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for _ in range(3):  # several rounds so that the two calls really overlap
        outs = []
        for d, st in zip(dev, streams):
            with torch.cuda.stream(st):
                outs.append(ag.ag_attn_fwd(d["q"], d["k"], d["v"], d["bias"], cap=5.0,
                                           stream=st))
    torch.cuda.synchronize()
    assert ag.ag_device_error(0) == 0
    for n, (c, (o, l)) in enumerate(zip(cases, outs)):
        B = c["q"].shape[0]
        rows = ag_inputs.sample_rows(B, 8, 8192, 256, seed=70 + n).numpy()
        ro, rl = oracle_lib.attn_rows(c["q"], c["k"], c["v"], c["bias"], rows, block=16,
                                      cap=5.0)
        b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
        on, ln = o.double().cpu().numpy(), l.double().cpu().numpy()
        _compare(on[b, h, i], ln[b, h, i], ro, rl, f"stream {n} B={B}")


@pytest.mark.parametrize("starts", [(0, 1024), (0, 704, 1408)])
def test_query_slabs_reproduce_the_full_call(ag, starts):
    """Queries split into slabs (ag_attn_fwd_query_slab: the slab's q rows and
    its bias rows, all keys): at L = 2048, B = 2 every call runs whole pairs of
    query blocks, so each slab's rows equal the full call's bit for bit."""
    B, L = 2, 2048
    inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=41, batched_bias=True)
    q, k, v, bias = (_dev(inp[n]) for n in ("q", "k", "v", "bias"))
    out, lse = ag.ag_attn_fwd(q, k, v, bias, cap=5.0)
    ends = starts[1:] + (L,)
    for q0, q1 in zip(starts, ends):
        so, sl = ag.ag_attn_fwd_query_slab(q[:, :, q0:q1].contiguous(), k, v,
                                           bias[:, :, q0 // 16:-(-q1 // 16)].contiguous(),
                                           cap=5.0)
        torch.cuda.synchronize()
        assert torch.equal(so, out[:, :, q0:q1]) and torch.equal(sl, lse[:, :, q0:q1]), \
            f"slab [{q0}, {q1}) differs from the full call"
    assert ag.ag_device_error(0) == 0


def test_query_slabs_full_context(ag, oracle_lib):
    """L = 8192 split into four slabs of 2048 queries, as four GPUs would hold
    them: every slab against the oracle on sampled rows."""
    L = 8192
    inp = ag_inputs.random_case(1, 8, L, 128, 128, 16, seed=43)
    q, k, v, bias = (_dev(inp[n]) for n in ("q", "k", "v", "bias"))
    for r in range(4):
        q0, q1 = 2048 * r, 2048 * (r + 1)
        so, sl = ag.ag_attn_fwd_query_slab(q[:, :, q0:q1].contiguous(), k, v,
                                           bias[:, q0 // 16:q1 // 16].contiguous(), cap=5.0)
        torch.cuda.synchronize()
        rows = ag_inputs.sample_rows(1, 8, 2048, 96, seed=r).numpy()
        glob = rows.copy()
        glob[:, 2] += q0
        ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], inp["bias"], glob,
                                      block=16, cap=5.0)
        b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
        _compare(so.double().cpu().numpy()[b, h, i], sl.double().cpu().numpy()[b, h, i],
                 ro, rl, f"slab {r} of L=8192")
    assert ag.ag_device_error(0) == 0


def test_maximum_length_sampled(ag, oracle_lib):
    inp = ag_inputs.random_case(1, 8, 65536, 128, 128, 16, seed=5)
    out, lse = _gpu_attn(ag, inp, 5.0)
    rows = ag_inputs.sample_rows(1, 8, 65536, 48, seed=3).numpy()
    ro, rl = oracle_lib.attn_rows(inp["q"], inp["k"], inp["v"], inp["bias"], rows,
                                  block=16, cap=5.0)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    _compare(out[b, h, i], lse[b, h, i], ro, rl, "L=65536 sampled")


def test_empty_inputs_are_noops(ag):
    q = torch.empty(0, 8, 64, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(0, 64, 128, dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(8, 4, 4, device="cuda")
    out, lse = ag.ag_attn_fwd(q, k, k, bias)
    assert out.shape == (0, 8, 64, 128) and lse.shape == (0, 8, 64)
    q0 = torch.empty(1, 8, 0, 128, dtype=torch.bfloat16, device="cuda")
    k0 = torch.empty(1, 0, 128, dtype=torch.bfloat16, device="cuda")
    ag.ag_attn_fwd(q0, k0, k0, torch.zeros(8, 0, 0, device="cuda"))
    pair = torch.empty(0, 0, 128, device="cuda")
    assert ag.ag_pair_bias_project(pair, torch.zeros(128, 8, device="cuda")).numel() == 0
    torch.cuda.synchronize()
    assert ag.ag_device_error(0) == 0


def test_deterministic_and_stream(ag):
    inp = ag_inputs.make_inputs(ag_inputs.WORKLOADS["short"])
    o1, l1 = _gpu_attn(ag, inp, 5.0)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = _gpu_attn(ag, inp, 5.0, stream=s)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


_MEMORY_PROBE = r"""
import json, sys, torch
sys.path.insert(0, sys.argv[1])
import ag_inputs
import long_context_genomics_b200 as ag
w = ag_inputs.WORKLOADS["full"]
inp = ag_inputs.make_inputs(w)
d = {n: t.cuda() for n, t in inp.items()}
bias = ag.ag_pair_bias_project(d["pair"], d["W"])   # loads the library's other modules
out = torch.empty(1, 8, w.L, 128, device="cuda")
lse = torch.empty(1, 8, w.L, device="cuda")
torch.cuda.synchronize()
free = [torch.cuda.mem_get_info()[0]]
for _ in range(2):
    ag.ag_attn_fwd(d["q"], d["k"], d["v"], bias, cap=5.0, out=out, lse=lse)
    torch.cuda.synchronize()
    free.append(torch.cuda.mem_get_info()[0])
assert ag.ag_device_error(0) == 0
print(json.dumps({"free": free, "lse0": float(lse[0, 0, 0])}))
"""


def test_no_quadratic_memory():
    """The attention allocates no device memory.  In a fresh process (so that
    the call is the first on the device), free device memory as the driver
    reports it (cudaMemGetInfo) before and after the first and the second
    call at L = 8192: the first call may only load the kernels' code (lazy
    module loading, well under 8 MiB; a single fp32 head of L x L logits
    would be 256 MiB, the old split-pair scratch 29 MB); the second changes
    nothing."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _MEMORY_PROBE, root], capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    rec = json.loads(res.stdout.strip().splitlines()[-1])
    f0, f1, f2 = rec["free"]
    print(f"free before {f0}, after first call {f1} (-{(f0 - f1) / 2**20:.2f} MiB), "
          f"after second {f2}")
    assert math.isfinite(rec["lse0"])
    assert 0 <= f0 - f1 <= 8 << 20
    assert f2 == f1


def test_bounded_wait_reports_and_context_survives(ag, oracle_lib):
    """A wait that nothing completes runs out after its limit, records
    (site 255 << 8) | 1 in the error word, and the context stays usable."""
    assert ag.ag_device_error(0) == 0
    ag.ag_debug_wait_timeout(20_000_000)
    code = ag.ag_device_error(0, clear=True)
    assert code == (255 << 8) | 1
    assert ag.ag_device_error(0) == 0
    inp = ag_inputs.random_case(1, 8, 256, 128, 128, 16, seed=9)
    out, lse = _gpu_attn(ag, inp, 5.0)
    ro, rl = oracle_lib.attn_fwd(inp["q"], inp["k"], inp["v"], inp["bias"],
                                 block=16, cap=5.0)
    _compare(out, lse, ro, rl, "after timeout")


def test_launch_count_matches_the_grid_policy(ag):
    """ag_attn_fwd_launch_count reports 1 or 2 kernels for real sizes and 0 for
    empty ones; at full context on a 148-SM B200 the 256 tile pairs do not
    divide evenly over the 74 SM pairs, so pairs are split and merged (2)."""
    assert ag.ag_attn_fwd_launch_count(0, 8192) == 0
    for B, L in [(1, 512), (1, 2048), (2, 8192)]:
        assert ag.ag_attn_fwd_launch_count(B, L) in (1, 2)
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert ag.ag_attn_fwd_launch_count(1, 8192) == 2
        # cap > 60 or none: the row maxima (split like the main kernel: two
        # launches) and the row-shift kernel on whole pairs.
        assert ag.ag_attn_fwd_launch_count(1, 8192, cap=math.inf) == 3
        assert ag.ag_attn_fwd_launch_count(1, 8192, cap=61.0) == 3
