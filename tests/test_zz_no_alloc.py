"""ag_attn_fwd_noalloc: the attention entry point that allocates nothing.

Some callers cannot let a library call cudaMalloc: code that must not touch
the allocator while a CUDA graph is being captured, or a framework that has
already handed all device memory to its own pool.  For them the library keeps
its split-pair scratch in a static device array instead of allocating it on
the first call.  This test calls that entry point through the C ABI and
checks it against ag_attn_fwd (which allocates its scratch) on two calls in a
row: a size that splits pairs between SMs (so the scratch is really used) and
then a different size, which must not be affected by what the first call left
in the shared static array.  This file sorts last so that a run stopping at
the first failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import ag_inputs

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_genomics_b200 as ag

    return ag.lib


def _call(fn, inp, cap):
    q, k, v, bias = (inp[n].cuda().contiguous() for n in ("q", "k", "v", "bias"))
    B, H, L, D = q.shape
    out = torch.full((B, H, L, D), float("nan"), device="cuda")
    lse = torch.full((B, H, L), float("nan"), device="cuda")
    st = fn(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(bias.data_ptr()),
            B, H, L, D, 16, ctypes.c_float(cap), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(lse.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, f"status {st}"
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


@pytest.mark.parametrize("cases", [[(1, 512, 5.0, 31), (1, 2064, math.inf, 32)]])
def test_noalloc_matches_allocating_entry_point(lib, cases):
    for B, L, cap, seed in cases:  # two calls in a row on the static scratch
        inp = ag_inputs.random_case(B, 8, L, 128, 128, 16, seed=seed)
        ref_out, ref_lse = _call(lib.ag_attn_fwd, inp, cap)
        out, lse = _call(lib.ag_attn_fwd_noalloc, inp, cap)
        assert np.isfinite(out).all() and np.isfinite(lse).all()
        eo = float(np.max(np.abs(out - ref_out)))
        el = float(np.max(np.abs(lse - ref_lse)))
        print(f"noalloc B={B} L={L} cap={cap}: max|dout|={eo:.3e} max|dlse|={el:.3e}")
        assert eo <= OUT_TOL and el <= LSE_TOL
