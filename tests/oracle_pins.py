"""Pins that tie the float64 oracle to things other than itself.

Each pin takes an ``oracle.Oracle`` handle and raises AssertionError when the
oracle disagrees with the mathematics of Eq. L_ij (page "Making Full-Context
AlphaGenome Fit on an RTX 3090", section "Why stock FlashAttention was not a
drop-in replacement") or of the pair projection (section "Profiling pointed at
one very large object").  They are run against the real oracle and against
builds with one planted mistake each (tests/test_oracle_mutants.py), which
every mistake must fail.

Kinds of pin used:
  * brute force on tiny inputs: a dense numpy evaluation that materialises
    the full L x L logits and the block-repeated bias with np.repeat;
  * special cases that reduce to a library routine: with cap = +inf the
    method is torch's scaled_dot_product_attention with the repeated bias as
    an additive mask;
  * closed forms: identical keys (uniform softmax, out = mean of V) and
    identical keys under a block bias (softmax over blocks);
  * invariances: key permutations inside a block, whole-block permutations
    carried into the bias columns, a constant bias shift (cap = +inf),
    equal heads, batch independence.
"""
from __future__ import annotations

import math

import numpy as np
import torch
from scipy.special import logsumexp

import ag_inputs

CAPS = (5.0, 30.0, math.inf)


def _case(B=2, H=3, L=64, D=8, Dv=6, block=16, seed=0, bias_std=1.0, qk_std=1.0,
          batched_bias=False):
    c = ag_inputs.random_case(B, H, L, D, Dv, block, seed, bias_std=bias_std,
                              qk_std=qk_std, dtype=torch.float64,
                              batched_bias=batched_bias)
    return {n: t.to(torch.float64).numpy() for n, t in c.items()}


def dense_bruteforce(q, k, v, bias, block, cap):
    """Dense evaluation with the literal block repeat of the compact bias,
    cropped to L when L is not a multiple of the block.  bias is [H,P,P], or
    [B,H,P,P] with one bias per batch item."""
    D = q.shape[-1]
    L = q.shape[2]
    b4 = bias if bias.ndim == 4 else bias[None]
    bexp = np.repeat(np.repeat(b4, block, axis=2), block, axis=3)[:, :, :L, :L]
    s = np.einsum("bhid,bjd->bhij", q, k) / np.sqrt(D) + bexp
    logits = s if math.isinf(cap) else cap * np.tanh(s / cap)
    lse = logsumexp(logits, axis=-1)
    p = np.exp(logits - lse[..., None])
    out = np.einsum("bhij,bjc->bhic", p, v)
    return out, lse, p


def _close(a, b, tol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max |diff| {err:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------
def pin_bruteforce(o):
    """Oracle == dense brute force on tiny inputs, several blocks and caps."""
    for block in (1, 2, 4, 16):
        for cap in CAPS:
            c = _case(L=64, block=block, seed=block)
            out, lse, p = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"],
                                     block=block, cap=cap, probs=True)
            ro, rl, rp = dense_bruteforce(c["q"], c["k"], c["v"], c["bias"], block, cap)
            _close(out, ro, 1e-12, f"out block={block} cap={cap}")
            _close(lse, rl, 1e-12, f"lse block={block} cap={cap}")
            _close(p, rp, 1e-12, f"probs block={block} cap={cap}")


def pin_bruteforce_tails_and_batched_bias(o):
    """Oracle == dense brute force for lengths that end in a partial block
    and for one bias per batch item."""
    for L, block in ((40, 16), (23, 4), (17, 16)):
        for cap in CAPS:
            for batched in (False, True):
                c = _case(B=3, L=L, block=block, seed=L + block, batched_bias=batched)
                out, lse, p = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"],
                                         block=block, cap=cap, probs=True)
                ro, rl, rp = dense_bruteforce(c["q"], c["k"], c["v"], c["bias"],
                                              block, cap)
                what = f"L={L} block={block} cap={cap} batched={batched}"
                _close(out, ro, 1e-12, "out " + what)
                _close(lse, rl, 1e-12, "lse " + what)
                _close(p, rp, 1e-12, "probs " + what)
    # Rows of a batched-bias case agree with the full evaluation.
    c = _case(B=2, L=40, block=16, seed=3, batched_bias=True)
    out, lse = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"], block=16, cap=5.0)
    rows = [[0, 0, 0], [1, 2, 39], [1, 0, 33], [0, 1, 16]]
    ro, rl = o.attn_rows(c["q"], c["k"], c["v"], c["bias"], rows, block=16, cap=5.0)
    for t, (b, h, i) in enumerate(rows):
        _close(ro[t], out[b, h, i], 1e-13, f"row {b},{h},{i} out")
        _close(rl[t], lse[b, h, i], 1e-13, f"row {b},{h},{i} lse")


def pin_sdpa(o):
    """cap = +inf reduces to scaled-dot-product attention with the repeated
    bias as an additive float mask (torch SDPA, float64, CPU)."""
    for bias_scale in (0.0, 1.0):
        c = _case(B=2, H=4, L=48, D=16, Dv=16, block=16, seed=7)
        bias = c["bias"] * bias_scale
        out, lse = o.attn_fwd(c["q"], c["k"], c["v"], bias, block=16, cap=math.inf)
        q = torch.from_numpy(c["q"])
        B, H, L, D = q.shape
        k = torch.from_numpy(c["k"])[:, None].expand(B, H, L, D)
        v = torch.from_numpy(c["v"])[:, None].expand(B, H, L, c["v"].shape[-1])
        mask = torch.from_numpy(bias).repeat_interleave(16, 1).repeat_interleave(16, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=mask[None].expand(B, H, L, L))
        _close(out, ref.numpy(), 1e-12, f"sdpa out (bias*{bias_scale})")
        logits = (q @ k.transpose(-1, -2)) / math.sqrt(D) + mask[None]
        _close(lse, torch.logsumexp(logits, -1).numpy(), 1e-12, "sdpa lse")


def pin_identical_keys(o):
    """All keys equal, bias 0: every logit in a row is cap*tanh(c_i/cap), so
    the softmax is uniform: out_i = mean_j v_j, lse_i = cap*tanh(c_i/cap) + ln L."""
    rng = np.random.default_rng(11)
    B, H, L, D, Dv = 1, 2, 64, 8, 5
    q = rng.normal(size=(B, H, L, D)) * 3.0
    k = np.broadcast_to(rng.normal(size=(1, 1, D)), (B, L, D)).copy()
    v = rng.normal(size=(B, L, Dv))
    bias = np.zeros((H, L // 16, L // 16))
    for cap in (5.0, 2.0):
        out, lse = o.attn_fwd(q, k, v, bias, block=16, cap=cap)
        c = np.einsum("bhid,d->bhi", q, k[0, 0]) / math.sqrt(D)
        want_lse = np.vectorize(lambda x: cap * math.tanh(x / cap))(c) + math.log(L)
        _close(lse, want_lse, 1e-12, f"identical-keys lse cap={cap}")
        want_out = np.broadcast_to(v.mean(axis=1)[:, None, None, :], out.shape)
        _close(out, want_out, 1e-12, f"identical-keys out cap={cap}")


def pin_block_bias_closed_form(o):
    """All keys equal, block-structured bias: key block J gets weight
    w_J = exp(cap*tanh((c_i + b[h,I,J])/cap)) shared by its `block` keys, so
    lse_i = ln(block * sum_J w_J) and out_i = sum_J w_J/sum(w) * mean(v in J).
    This fixes the bias orientation (row = query block, column = key block),
    the floor indexing, and the bias-inside-the-cap order."""
    rng = np.random.default_rng(5)
    B, H, L, D, Dv, blk = 1, 2, 64, 4, 3, 16
    P = L // blk
    q = rng.normal(size=(B, H, L, D)) * 2.0
    k = np.broadcast_to(rng.normal(size=(1, 1, D)), (B, L, D)).copy()
    v = rng.normal(size=(B, L, Dv))
    bias = rng.normal(size=(H, P, P)) * 2.0
    for cap in (5.0, 1.5):
        out, lse = o.attn_fwd(q, k, v, bias, block=blk, cap=cap)
        vbar = v[0].reshape(P, blk, Dv).mean(axis=1)  # [P, Dv]
        for h in range(H):
            for i in range(L):
                c = float(q[0, h, i] @ k[0, 0]) / math.sqrt(D)
                I = i // blk
                w = np.array([math.exp(cap * math.tanh((c + bias[h, I, J]) / cap))
                              for J in range(P)])
                assert abs(lse[0, h, i] - math.log(blk * w.sum())) <= 1e-12, \
                    f"block-bias lse h={h} i={i}"
                want = (w / w.sum()) @ vbar
                _close(out[0, h, i], want, 1e-12, f"block-bias out h={h} i={i}")


def pin_cap_limit(o):
    """A very large cap approaches no cap: cap*tanh(s/cap) = s - s^3/(3cap^2)+..."""
    c = _case(L=32, block=16, seed=3)
    o1, l1 = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"], block=16, cap=1e6)
    o2, l2 = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"], block=16, cap=math.inf)
    _close(o1, o2, 1e-9, "cap->inf out")
    _close(l1, l2, 1e-9, "cap->inf lse")


def pin_probabilities(o):
    """Softmax rows sum to 1, out = P @ V, and lse is log-sum-exp of the
    logits recovered from P (log p + lse equal per row up to a shift)."""
    c = _case(L=32, block=16, seed=4)
    out, lse, p = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"], block=16,
                             cap=5.0, probs=True)
    _close(p.sum(-1), np.ones(p.shape[:-1]), 1e-13, "prob rows sum")
    assert (p > 0).all(), "probabilities must be positive"
    _close(out, np.einsum("bhij,bjc->bhic", p, c["v"]), 1e-12, "out = P V")
    # The capped logits are bounded by cap, so lse <= cap + ln L.
    assert (lse <= 5.0 + math.log(32) + 1e-12).all(), "lse above cap + ln L"


def pin_invariances(o):
    """Symmetries of the definition."""
    c = _case(B=2, H=2, L=64, D=8, Dv=4, block=16, seed=9)
    q, k, v, bias = c["q"], c["k"], c["v"], c["bias"]
    base_o, base_l = o.attn_fwd(q, k, v, bias, block=16, cap=5.0)
    rng = np.random.default_rng(1)
    # (a) permuting keys (with their values) inside each block
    perm = np.concatenate([J * 16 + rng.permutation(16) for J in range(4)])
    o1, l1 = o.attn_fwd(q, k[:, perm], v[:, perm], bias, block=16, cap=5.0)
    _close(o1, base_o, 1e-12, "perm within block out")
    _close(l1, base_l, 1e-12, "perm within block lse")
    # (b) permuting whole key blocks together with the bias columns
    bperm = np.array([2, 0, 3, 1])
    kperm = np.concatenate([np.arange(16) + 16 * J for J in bperm])
    o2, l2 = o.attn_fwd(q, k[:, kperm], v[:, kperm], bias[:, :, bperm],
                        block=16, cap=5.0)
    _close(o2, base_o, 1e-12, "block perm out")
    _close(l2, base_l, 1e-12, "block perm lse")
    # (c) a constant bias shift with no cap: out unchanged, lse shifted
    oi, li = o.attn_fwd(q, k, v, bias, block=16, cap=math.inf)
    o3, l3 = o.attn_fwd(q, k, v, bias + 0.75, block=16, cap=math.inf)
    _close(o3, oi, 1e-12, "shift out")
    _close(l3, li + 0.75, 1e-12, "shift lse")
    # (d) equal queries and bias on every head give equal rows on every head
    qe = np.repeat(q[:, :1], 2, axis=1)
    be = np.repeat(bias[:1], 2, axis=0)
    o4, l4 = o.attn_fwd(qe, k, v, be, block=16, cap=5.0)
    _close(o4[:, 0], o4[:, 1], 0.0, "equal heads out")
    _close(l4[:, 0], l4[:, 1], 0.0, "equal heads lse")
    # (e) each batch item alone gives the same rows
    for b in range(2):
        o5, l5 = o.attn_fwd(q[b:b + 1], k[b:b + 1], v[b:b + 1], bias, block=16, cap=5.0)
        _close(o5[0], base_o[b], 0.0, f"batch {b} out")
        _close(l5[0], base_l[b], 0.0, f"batch {b} lse")
    # (f) permuting queries inside a block permutes the output rows
    qp = np.concatenate([J * 16 + rng.permutation(16) for J in range(4)])
    o6, l6 = o.attn_fwd(q[:, :, qp], k, v, bias, block=16, cap=5.0)
    _close(o6, base_o[:, :, qp], 1e-12, "query perm out")
    _close(l6, base_l[:, :, qp], 1e-12, "query perm lse")


def pin_rows(o):
    """The row-sampled entry point returns exactly the matching full rows."""
    c = _case(B=2, H=3, L=64, D=8, Dv=6, block=16, seed=12)
    out, lse = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"], block=16, cap=5.0)
    rows = np.array([[0, 0, 0], [1, 2, 63], [0, 1, 17], [1, 0, 40]])
    ro, rl = o.attn_rows(c["q"], c["k"], c["v"], c["bias"], rows, block=16, cap=5.0)
    for t, (b, h, i) in enumerate(rows):
        _close(ro[t], out[b, h, i], 0.0, f"row {t} out")
        _close(rl[t], lse[b, h, i], 0.0, f"row {t} lse")


def pin_projection(o):
    """Pair projection: one-hot W columns pick a channel (fixes the [H,P,P]
    orientation and the W[c,h] indexing), a constant pair gives the column
    sums of W, the map is linear in W, and it equals numpy's einsum of the
    same contraction."""
    rng = np.random.default_rng(2)
    P, Cp, H = 6, 5, 3
    pair = rng.normal(size=(P, P, Cp))
    W = np.zeros((Cp, H))
    chans = [4, 0, 2]
    for h, c in enumerate(chans):
        W[c, h] = 1.0
    b = o.pair_bias_project(pair, W)
    for h, c in enumerate(chans):
        _close(b[h], pair[:, :, c], 0.0, f"one-hot channel {c}")
    W2 = rng.normal(size=(Cp, H))
    b2 = o.pair_bias_project(np.full((P, P, Cp), 0.5), W2)
    want = np.broadcast_to((0.5 * W2.sum(axis=0))[:, None, None], (H, P, P))
    _close(b2, want, 1e-14, "constant pair")
    W3 = rng.normal(size=(Cp, H))
    lin = o.pair_bias_project(pair, W2 + W3)
    _close(lin, o.pair_bias_project(pair, W2) + o.pair_bias_project(pair, W3),
           1e-12, "linearity")
    # A library contraction of the same definition (numpy einsum).
    _close(o.pair_bias_project(pair, W3), np.einsum("pqc,ch->hpq", pair, W3), 1e-12,
           "einsum")


# ---- backward ---------------------------------------------------------------
def torch_dense_grads(q, k, v, bias, dout, block, cap):
    """Gradients of sum(out * dout) by torch autograd (float64, CPU) through a
    dense evaluation of its own: the compact bias is repeated with
    repeat_interleave, so its gradient is autograd's sum over each cell."""
    t = {n: torch.tensor(x, dtype=torch.float64, requires_grad=True)
         for n, x in (("q", q), ("k", k), ("v", v), ("bias", bias))}
    L, D = q.shape[2], q.shape[3]
    b4 = t["bias"] if bias.ndim == 4 else t["bias"][None]
    bexp = b4.repeat_interleave(block, 2).repeat_interleave(block, 3)[:, :, :L, :L]
    s = torch.einsum("bhid,bjd->bhij", t["q"], t["k"]) / math.sqrt(D) + bexp
    logits = s if math.isinf(cap) else cap * torch.tanh(s / cap)
    out = torch.einsum("bhij,bjc->bhic", torch.softmax(logits, -1), t["v"])
    (out * torch.from_numpy(dout)).sum().backward()
    return [t[n].grad.numpy() for n in ("q", "k", "v", "bias")]


def _bwd_case(B=2, H=3, L=40, D=8, Dv=6, block=16, seed=0, batched_bias=False):
    c = _case(B=B, H=H, L=L, D=D, Dv=Dv, block=block, seed=seed, batched_bias=batched_bias)
    c["dout"] = np.random.default_rng(seed + 100).normal(size=(B, H, L, Dv))
    return c


def pin_bwd_autograd(o):
    """Oracle gradients == torch autograd of a dense evaluation, for several
    blocks and caps, a partial last block, a bias shared by two items (its
    gradient sums over them) and one bias per item."""
    cases = [dict(L=64, block=16), dict(L=40, block=16), dict(L=23, block=4),
             dict(L=32, block=1), dict(L=48, block=16, batched_bias=True)]
    for n, kw in enumerate(cases):
        for cap in CAPS:
            c = _bwd_case(seed=n, **kw)
            got = o.attn_bwd(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                             block=kw["block"], cap=cap)
            want = torch_dense_grads(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                                     kw["block"], cap)
            for name, g, w in zip(("dq", "dk", "dv", "dbias"), got[:4], want):
                _close(g, w, 1e-11, f"{name} {kw} cap={cap}")


def pin_bwd_finite_differences(o):
    """Directional derivatives of f = sum(out * dout) by central differences of
    the forward oracle match the backward oracle's gradients."""
    c = _bwd_case(B=2, H=2, L=40, D=8, Dv=5, block=16, seed=21)
    rng = np.random.default_rng(22)
    for cap in (5.0, math.inf):
        dq, dk, dv, db, _, _ = o.attn_bwd(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                                          block=16, cap=cap)
        grads = {"q": dq, "k": dk, "v": dv, "bias": db}
        for name in ("q", "k", "v", "bias"):
            u = rng.normal(size=c[name].shape)
            eps = 1e-5

            def f(sign):
                x = dict(c)
                x[name] = c[name] + sign * eps * u
                out, _ = o.attn_fwd(x["q"], x["k"], x["v"], x["bias"], block=16, cap=cap)
                return float(np.sum(out * c["dout"]))

            fd = (f(+1) - f(-1)) / (2 * eps)
            an = float(np.sum(grads[name] * u))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), \
                f"d/d{name} cap={cap}: finite difference {fd:.10g} vs gradient {an:.10g}"


def pin_bwd_closed_forms(o):
    """(a) All keys equal and no bias: the softmax is uniform and its logits
    are equal, so dq = 0 and dv_j = (1/L) sum_{h,i} dout_i for every key.
    (b) No cap: adding a constant to one query block's bias row changes
    nothing, so each row of dbias sums to 0 over the key blocks.
    (c) delta_i = dout_i . out_i (sum_j p_ij v_j = out_i)."""
    rng = np.random.default_rng(31)
    B, H, L, D, Dv = 1, 2, 48, 8, 5
    q = rng.normal(size=(B, H, L, D)) * 2.0
    k = np.broadcast_to(rng.normal(size=(1, 1, D)), (B, L, D)).copy()
    v = rng.normal(size=(B, L, Dv))
    dout = rng.normal(size=(B, H, L, Dv))
    bias = np.zeros((H, L // 16, L // 16))
    for cap in (5.0, math.inf):
        dq, _, dv, _, _, _ = o.attn_bwd(q, k, v, bias, dout, block=16, cap=cap)
        _close(dq, np.zeros_like(dq), 1e-12, f"identical keys dq cap={cap}")
        want = np.broadcast_to(dout.sum(axis=(1, 2))[:, None, :] / L, dv.shape)
        _close(dv, want, 1e-12, f"identical keys dv cap={cap}")
    c = _bwd_case(B=2, H=3, L=40, D=8, Dv=6, block=16, seed=32)
    _, _, _, db, _, delta = o.attn_bwd(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                                       block=16, cap=math.inf)
    _close(db.sum(axis=-1), np.zeros(db.shape[:-1]), 1e-12, "no-cap dbias row sums")
    out, _ = o.attn_fwd(c["q"], c["k"], c["v"], c["bias"], block=16, cap=5.0)
    _, _, _, _, _, delta5 = o.attn_bwd(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                                       block=16, cap=5.0)
    _close(delta5, np.einsum("bhic,bhic->bhi", c["dout"], out), 1e-12, "delta = dout . out")


def pin_bwd_sample(o):
    """The sampled backward entry returns exactly the full backward's values,
    for a shared bias (cells summed over the items) and one bias per item."""
    for batched in (False, True):
        c = _bwd_case(B=2, H=3, L=40, D=8, Dv=6, block=16, seed=41, batched_bias=batched)
        dq, dk, dv, db, _, _ = o.attn_bwd(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                                          block=16, cap=5.0)
        rows = [[0, 0, 0], [1, 2, 39], [0, 1, 17]]
        keys = [[0, 0], [1, 39], [1, 16]]
        cells = [[0, 0, 0, 0], [1, 2, 2, 1], [1, 1, 0, 2]]
        sq, sk, sv, sb = o.attn_bwd_sample(c["q"], c["k"], c["v"], c["bias"], c["dout"],
                                           rows=rows, keys=keys, cells=cells,
                                           block=16, cap=5.0)
        for t, (b, h, i) in enumerate(rows):
            _close(sq[t], dq[b, h, i], 1e-13, f"sample dq {b},{h},{i}")
        for t, (b, j) in enumerate(keys):
            _close(sk[t], dk[b, j], 1e-13, f"sample dk {b},{j}")
            _close(sv[t], dv[b, j], 1e-13, f"sample dv {b},{j}")
        for t, (b, h, I, J) in enumerate(cells):
            want = db[b, h, I, J] if batched else db[h, I, J]
            _close(sb[t], want, 1e-13, f"sample dbias {b},{h},{I},{J}")


ALL_PINS = [
    pin_bruteforce, pin_bruteforce_tails_and_batched_bias, pin_sdpa, pin_identical_keys, pin_block_bias_closed_form,
    pin_cap_limit, pin_probabilities, pin_invariances, pin_rows, pin_projection,
    pin_bwd_autograd, pin_bwd_finite_differences, pin_bwd_closed_forms, pin_bwd_sample,
]
