"""The C ABI without a GPU: libag loads, exports every function that
include/ag.h declares, and rejects bad arguments with the documented status
before touching CUDA.  No call here reaches a kernel launch."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ag.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ag_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def ag():
    import long_context_genomics_b200 as ag

    return ag


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("ag_pair_bias_project", "ag_attn_fwd", "ag_status_string",
                     "ag_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(ag):
    lib = ctypes.CDLL(ag.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, f"declared in ag.h but not exported: {missing}"


def test_status_strings(ag):
    for code, name in ag.STATUS_NAMES.items():
        assert ag.ag_status_string(code).startswith(name)
    assert "unknown" in ag.ag_status_string(99)
    assert ag.ag_version() >= 100


# Fake, never-dereferenced device addresses: validation fails before CUDA.
A16 = 0x10000
BAD = 0x10004  # 4-byte aligned, not 16


def _attn(ag, q=A16, k=A16 * 2, v=A16 * 3, bias=A16 * 4, B=1, H=8, L=256, D=128,
          block=16, cap=5.0, out=A16 * 1000, lse=A16 * 2000):
    return ag.lib.ag_attn_fwd(q, k, v, bias, B, H, L, D, block, cap, out, lse, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(lse=None), 1), (dict(bias=None), 1),
    (dict(B=-1), 2), (dict(L=-16), 2), (dict(D=0), 2),
    (dict(H=4), 4), (dict(D=64), 4), (dict(block=8), 4), (dict(L=65536 + 16), 4),
    (dict(B=1 << 20, L=65536), 4),
    # B * L = 2^27 is allowed, but B * ceil(L/32) * ceil(L/128) = 2^31 work steps is not.
    (dict(B=2048, L=65536), 4), (dict(B=1024, L=65536, q=None), 1),
    (dict(cap=0.0), 5), (dict(cap=-1.0), 5), (dict(cap=math.nan), 5),
    (dict(q=BAD), 3), (dict(k=BAD), 3), (dict(out=BAD), 3),
    (dict(out=A16), 7), (dict(lse=A16 * 4), 7),
])
def test_attn_validation(ag, kw, status):
    assert _attn(ag, **kw) == status


def test_launch_count_checks_before_the_device(ag):
    import ctypes
    n = ctypes.c_int(-1)
    f = ag.lib.ag_attn_fwd_launch_count
    assert f(1, 8, 256, 128, 16, 5.0, None) == 1                    # AG_ERR_NULL
    assert f(1, 8, -1, 128, 16, 5.0, ctypes.byref(n)) == 2          # AG_ERR_SHAPE
    assert f(1, 8, 256, 64, 16, 5.0, ctypes.byref(n)) == 4          # AG_ERR_UNSUPPORTED
    assert f(1, 8, 256, 128, 16, -1.0, ctypes.byref(n)) == 5        # AG_ERR_VALUE
    assert f(0, 8, 256, 128, 16, 5.0, ctypes.byref(n)) == 0 and n.value == 0


def _attn_strided(ag, stride, q=A16, k=A16 * 2, v=A16 * 3, bias=A16 * 4, B=2, H=8,
                  L=250, D=128, block=16, cap=5.0, out=A16 * 1000, lse=A16 * 2000):
    return ag.lib.ag_attn_fwd_strided_bias(q, k, v, bias, stride, B, H, L, D, block,
                                           cap, out, lse, None)


def test_strided_bias_validation(ag):
    # L = 250 ends in a partial block: P = 16 cells per side.
    P = 16
    assert _attn_strided(ag, -1) == 2                      # negative stride
    assert _attn_strided(ag, 8 * P * P - 1) == 2           # overlapping items
    assert _attn_strided(ag, 8 * P * P, q=None) == 1       # a dense [B,H,P,P]: passes to NULL check
    assert _attn_strided(ag, 0, q=None) == 1               # shared bias
    assert _attn_strided(ag, 8 * P * P, bias=BAD + 1) == 3  # bias not 4-byte aligned
    # The per-item bias span (B-1)*stride + H*P*P floats must not overlap out.
    span = (1 * 10 * 8 * P * P + 8 * P * P) * 4
    assert _attn_strided(ag, 10 * 8 * P * P, bias=A16 * 1000 - span + 16) == 7
    # A span beyond 2^56 floats is refused before its size can overflow.
    assert _attn_strided(ag, 1 << 62, q=None) == 2
    assert _attn_strided(ag, (1 << 56) // 9, B=10, q=None) == 2
    assert _attn_strided(ag, (1 << 56) // 10, B=10, q=None) == 1


def test_value_width_validation(ag):
    f = ag.lib.ag_attn_fwd_ex
    args = lambda Dv, **kw: (kw.get("q", A16), A16 * 2, A16 * 3, A16 * 4, 0, 1, 8, 256,
                             128, Dv, 16, 5.0, A16 * 1000, A16 * 2000, None)
    assert f(*args(0)) == 2          # AG_ERR_SHAPE
    assert f(*args(64)) == 4         # AG_ERR_UNSUPPORTED
    assert f(*args(160)) == 4
    assert f(*args(192, q=None)) == 1  # supported width: on to the NULL check
    assert f(*args(128, q=None)) == 1


def test_attn_empty_is_a_noop(ag):
    assert _attn(ag, B=0, q=None, k=None, v=None, bias=None, out=None, lse=None) == 0
    assert _attn(ag, L=0, q=None, k=None, v=None, bias=None, out=None, lse=None) == 0


@pytest.mark.parametrize("args,status", [
    ((A16, A16 * 2, A16 * 3, -1, 128, 8), 2),
    ((A16, A16 * 2, A16 * 3, 16, 0, 8), 2),
    ((A16, A16 * 2, A16 * 3, 16, 64, 8), 4),
    ((A16, A16 * 2, A16 * 3, 16, 128, 4), 4),
    ((A16, A16 * 2, A16 * 3, 8192, 128, 8), 4),
    ((None, A16 * 2, A16 * 3, 16, 128, 8), 1),
    ((BAD, A16 * 2, A16 * 3, 16, 128, 8), 3),
    ((A16, A16 * 2, A16 + 64, 16, 128, 8), 7),
    ((0, 0, 0, 0, 128, 8), 0),
])
def test_projection_validation(ag, args, status):
    assert ag.lib.ag_pair_bias_project(*args, None) == status


def test_binding_rejects_cpu_tensors(ag):
    import torch

    q = torch.zeros(1, 8, 16, 128, dtype=torch.bfloat16)
    k = torch.zeros(1, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ag.ag_attn_fwd(q, k, k, torch.zeros(8, 1, 1))


def test_binding_refuses_tensors_on_different_devices(ag):
    import torch

    a, b = torch.zeros(2), torch.zeros(2, device="meta")
    assert ag._one_device(a, torch.ones(3)) == torch.device("cpu")
    with pytest.raises(ValueError, match="must be on"):
        ag._one_device(a, b)


def _bwd(ag, q=A16, k=A16 * 2, v=A16 * 3, bias=A16 * 4, stride=0, lse=A16 * 5,
         dout=A16 * 6, B=1, H=8, L=256, D=128, Dv=128, block=16, cap=5.0,
         dq=A16 * 1000, dk=A16 * 2000, dv=A16 * 3000, dbias=A16 * 4000, delta=A16 * 5000):
    return ag.lib.ag_attn_bwd(q, k, v, bias, stride, lse, dout, B, H, L, D, Dv, block,
                              cap, dq, dk, dv, dbias, delta, None)


def test_backward_validation(ag):
    assert _bwd(ag, L=-1) == 2                    # AG_ERR_SHAPE
    assert _bwd(ag, D=64) == 4                    # AG_ERR_UNSUPPORTED
    assert _bwd(ag, H=4) == 4
    assert _bwd(ag, cap=float("nan")) == 5        # AG_ERR_VALUE
    assert _bwd(ag, cap=0.0) == 5
    assert _bwd(ag, Dv=0) == 2
    assert _bwd(ag, Dv=96) == 4
    assert _bwd(ag, stride=-1) == 2
    assert _bwd(ag, stride=8 * 16 * 16 - 1) == 2  # items' bias would overlap
    assert _bwd(ag, B=0, q=None, dq=None) == 0    # empty: a no-op
    assert _bwd(ag, L=0, dout=None) == 0
    for name in ("q", "k", "v", "bias", "lse", "dout", "dq", "dk", "dv", "dbias", "delta"):
        assert _bwd(ag, **{name: None}) == 1, name  # AG_ERR_NULL
    assert _bwd(ag, q=A16 + 1) == 3               # bf16 needs 2-byte alignment
    assert _bwd(ag, lse=A16 + 2) == 3             # fp32 needs 4-byte alignment
    # Value width 128 (the tensor-core path): q, k, v, dout, dq 16-byte aligned.
    for name in ("q", "k", "v", "dout", "dq"):
        assert _bwd(ag, **{name: (A16 * 6 if name == "dout" else
                                  A16 * 1000 if name == "dq" else
                                  A16 * {"q": 1, "k": 2, "v": 3}[name]) + 4}) == 3, name
    # Outputs overlapping an input or one another.
    assert _bwd(ag, dq=A16 * 6) == 7              # dq on dout
    assert _bwd(ag, delta=A16 * 1000 + 64) == 7   # delta inside dq
    assert _bwd(ag, dbias=A16 * 4) == 7           # dbias on bias


def test_backward_launch_count(ag):
    n = ctypes.c_int(-1)
    assert ag.lib.ag_attn_bwd_launch_count(128, ctypes.byref(n)) == 0 and n.value == 4
    assert ag.lib.ag_attn_bwd_launch_count(192, ctypes.byref(n)) == 0 and n.value == 2
    assert ag.lib.ag_attn_bwd_launch_count(128, None) == 1   # AG_ERR_NULL
    assert ag.lib.ag_attn_bwd_launch_count(0, ctypes.byref(n)) == 2
    assert ag.lib.ag_attn_bwd_launch_count(96, ctypes.byref(n)) == 4
    assert ag.ag_attn_bwd_launch_count() == 4 and ag.ag_attn_bwd_launch_count(192) == 2
