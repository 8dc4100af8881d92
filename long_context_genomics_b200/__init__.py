"""Python binding of libag: pair-bias multi-query attention on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels of libag.so (see include/ag.h for the C ABI); there is no CPU or
PyTorch fallback, and importing this package raises if the library is
missing.  PyTorch supplies device memory and the current stream.

    ag_pair_bias_project(pair[P,P,Cp] f32, W[Cp,H] f32) -> bias[H,P,P] f32
    ag_attn_fwd(q[B,H,L,D] bf16, k[B,L,D] bf16, v[B,L,D] bf16,
                bias[H,P,P] f32, cap) -> (out[B,H,L,D] f32, lse[B,H,L] f32)

The operation is Eq. L_ij of the page "Making Full-Context AlphaGenome Fit
on an RTX 3090" (section "Why stock FlashAttention was not a drop-in
replacement") with a softmax over all keys.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libag.so")

AG_OK = 0
STATUS_NAMES = {
    0: "AG_OK", 1: "AG_ERR_NULL", 2: "AG_ERR_SHAPE", 3: "AG_ERR_ALIGN",
    4: "AG_ERR_UNSUPPORTED", 5: "AG_ERR_VALUE", 6: "AG_ERR_CUDA",
    7: "AG_ERR_ALIAS", 8: "AG_ERR_DEVICE", 9: "AG_ERR_SCRATCH",
}


class AgError(RuntimeError):
    """A libag call returned a status other than AG_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {ag_status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python long_context_genomics_b200/build.py` (or __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
    lib.ag_status_string.argtypes = [ctypes.c_int]
    lib.ag_status_string.restype = ctypes.c_char_p
    lib.ag_version.argtypes = []
    lib.ag_version.restype = ctypes.c_int
    lib.ag_pair_bias_project.argtypes = [vp, vp, vp, i64, i64, i64, vp]
    lib.ag_pair_bias_project.restype = ctypes.c_int
    lib.ag_pair_bias_project_rows.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp]
    lib.ag_pair_bias_project_rows.restype = ctypes.c_int
    lib.ag_attn_fwd.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32,
                                vp, vp, vp]
    lib.ag_attn_fwd.restype = ctypes.c_int
    lib.ag_attn_fwd_strided_bias.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64,
                                             i64, i64, f32, vp, vp, vp]
    lib.ag_attn_fwd_strided_bias.restype = ctypes.c_int
    lib.ag_attn_fwd_ex.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64,
                                   i64, f32, vp, vp, vp]
    lib.ag_attn_fwd_ex.restype = ctypes.c_int
    lib.ag_attn_fwd_query_slab.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64,
                                           i64, i64, f32, vp, vp, vp]
    lib.ag_attn_fwd_query_slab.restype = ctypes.c_int
    lib.ag_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                        f32, vp, vp, vp]
    lib.ag_attn_fwd_noalloc.restype = ctypes.c_int
    lib.ag_attn_fwd_launch_count.argtypes = [i64, i64, i64, i64, i64, f32,
                                             ctypes.POINTER(ctypes.c_int)]
    lib.ag_attn_fwd_launch_count.restype = ctypes.c_int
    ip = ctypes.POINTER(ctypes.c_int)
    lib.ag_attn_fwd_schedule.argtypes = [i64, i64, ctypes.c_int, ctypes.c_int, ip, ip, ip,
                                         ip, ip, ip, ip, ip]
    lib.ag_attn_fwd_schedule.restype = ctypes.c_int
    lib.ag_attn_bwd.argtypes = [vp, vp, vp, vp, i64, vp, vp, i64, i64, i64, i64, i64,
                                i64, f32, vp, vp, vp, vp, vp, vp]
    lib.ag_attn_bwd.restype = ctypes.c_int
    lib.ag_attn_bwd_launch_count.argtypes = [i64, ctypes.POINTER(ctypes.c_int)]
    lib.ag_attn_bwd_launch_count.restype = ctypes.c_int
    lib.ag_device_error.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                    ctypes.c_int]
    lib.ag_device_error.restype = ctypes.c_int
    lib.ag_debug_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.ag_debug_wait_timeout.restype = ctypes.c_int
    return lib


lib = _load()


def ag_status_string(status: int) -> str:
    return lib.ag_status_string(int(status)).decode()


def ag_version() -> int:
    return int(lib.ag_version())


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _one_device(*tensors: torch.Tensor) -> torch.device:
    """The one device that every tensor of a call lives on.  The kernels run
    on that device (made current for the call), so a tensor elsewhere would
    reach them as a pointer they cannot read: refuse it here."""
    dev = tensors[0].device
    for t in tensors[1:]:
        if t.device != dev:
            raise ValueError(f"all tensors of a call must be on {dev}; one is on {t.device}")
    return dev


def _check(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def ag_pair_bias_project(pair: torch.Tensor, W: torch.Tensor,
                         bias: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bias[h,p,q] = sum_c pair[p,q,c] W[c,h] on the GPU (libag kernel)."""
    _check(pair, "pair", torch.float32, 3)
    _check(W, "W", torch.float32, 2)
    P, P2, Cp = pair.shape
    if P != P2 or W.shape[0] != Cp:
        raise ValueError("pair must be [P,P,Cp] and W [Cp,H]")
    H = W.shape[1]
    if bias is None:
        bias = torch.empty((H, P, P), dtype=torch.float32, device=pair.device)
    _check(bias, "bias", torch.float32, 3)
    if tuple(bias.shape) != (H, P, P):
        raise ValueError("bias must be [H,P,P]")
    with torch.cuda.device(_one_device(pair, W, bias)):
        st = lib.ag_pair_bias_project(pair.data_ptr(), W.data_ptr(), bias.data_ptr(),
                                      P, Cp, H, _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_pair_bias_project", st)
    return bias


def ag_pair_bias_project_rows(pair: torch.Tensor, W: torch.Tensor,
                              bias: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bias[h,r,q] = sum_c pair[r,q,c] W[c,h] for a row slab pair[R,P,Cp]
    (libag kernel); returns bias [H,R,P]."""
    _check(pair, "pair", torch.float32, 3)
    _check(W, "W", torch.float32, 2)
    R, P, Cp = pair.shape
    if W.shape[0] != Cp:
        raise ValueError("pair must be [R,P,Cp] and W [Cp,H]")
    H = W.shape[1]
    if bias is None:
        bias = torch.empty((H, R, P), dtype=torch.float32, device=pair.device)
    _check(bias, "bias", torch.float32, 3)
    if tuple(bias.shape) != (H, R, P):
        raise ValueError("bias must be [H,R,P]")
    with torch.cuda.device(_one_device(pair, W, bias)):
        st = lib.ag_pair_bias_project_rows(pair.data_ptr(), W.data_ptr(), bias.data_ptr(),
                                           R, P, Cp, H, _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_pair_bias_project_rows", st)
    return bias


def ag_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                bias: torch.Tensor, cap: float = 5.0, block: int = 16,
                out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                stream=None):
    """Fused pair-bias MQA attention forward (libag kernel).

    bias is [H,P,P] (shared by the batch) or [B,H,P,P] (one per batch item),
    P = ceil(L / block); v is [B,L,Dv] with Dv = D or 192 (the page's
    checkpoint).  Calls ag_attn_fwd_ex.  Returns (out [B,H,L,Dv] fp32,
    lse [B,H,L] fp32).  cap = math.inf turns the soft cap off."""
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    if tuple(k.shape) != (B, L, D) or tuple(v.shape) != (B, L, Dv):
        raise ValueError("k must be [B,L,D] and v [B,L,Dv] with q [B,H,L,D]")
    bstride = _bias_stride(bias, B, H, L, block)
    if out is None:
        out = torch.empty((B, H, L, Dv), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _check_out(out, lse, B, H, L, Dv)
    with torch.cuda.device(_one_device(q, k, v, bias, out, lse)):
        st = lib.ag_attn_fwd_ex(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), bias.data_ptr(), bstride, B, H, L,
            D, Dv, int(block), float(cap), out.data_ptr(), lse.data_ptr(),
            _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_attn_fwd_ex", st)
    return out, lse


def ag_attn_fwd_query_slab(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           bias: torch.Tensor, cap: float = 5.0, block: int = 16,
                           out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                           stream=None):
    """The attention rows of a slab of query positions (libag kernel).

    q [B,H,Lq,D] holds positions q0 .. q0+Lq-1 (q0 a multiple of block) of
    sequences whose keys and values k [B,L,D], v [B,L,Dv] are all given; bias
    holds the slab's bias rows, [H, ceil(Lq/block), ceil(L/block)] (shared by
    the batch) or [B, H, ceil(Lq/block), ceil(L/block)].  Returns
    (out [B,H,Lq,Dv] fp32, lse [B,H,Lq] fp32)."""
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    B, H, Lq, D = q.shape
    L, Dv = k.shape[1], v.shape[-1]
    if tuple(k.shape) != (B, L, D) or tuple(v.shape) != (B, L, Dv):
        raise ValueError("k must be [B,L,D] and v [B,L,Dv] with q [B,H,Lq,D]")
    bstride = _bias_stride(bias, B, H, L, block, rows=-(-Lq // block) if block > 0 else 0)
    if out is None:
        out = torch.empty((B, H, Lq, Dv), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    _check_out(out, lse, B, H, Lq, Dv)
    with torch.cuda.device(_one_device(q, k, v, bias, out, lse)):
        st = lib.ag_attn_fwd_query_slab(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), bias.data_ptr(), bstride, B, H, Lq, L,
            D, Dv, int(block), float(cap), out.data_ptr(), lse.data_ptr(),
            _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_attn_fwd_query_slab", st)
    return out, lse


def _bias_stride(bias: torch.Tensor, B: int, H: int, L: int, block: int,
                 rows: int | None = None) -> int:
    """Batch stride (floats) of a [H,R,P] (0) or [B,H,R,P] bias, P = ceil(L/block)
    and R = rows (default P)."""
    if bias.dtype != torch.float32 or not bias.is_contiguous():
        raise ValueError("bias must be a contiguous float32 tensor")
    P = -(-L // block) if block > 0 else 0
    R = P if rows is None else rows
    if tuple(bias.shape) == (H, R, P):
        return 0
    if tuple(bias.shape) == (B, H, R, P):
        return H * R * P
    raise ValueError(f"bias must be [{H},{R},{P}] or [{B},{H},{R},{P}], got {tuple(bias.shape)}")


def _check_out(out: torch.Tensor, lse: torch.Tensor, B: int, H: int, L: int, Dv: int):
    _check(out, "out", torch.float32, 4)
    _check(lse, "lse", torch.float32, 3)
    if tuple(out.shape) != (B, H, L, Dv) or tuple(lse.shape) != (B, H, L):
        raise ValueError("out must be [B,H,L,Dv] and lse [B,H,L]")


def ag_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        bias: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
                        cap: float = 5.0, block: int = 16, stream=None):
    """ag_attn_fwd through the entry point that allocates nothing (static
    scratch inside the library).  The caller passes the outputs."""
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check(bias, "bias", torch.float32, 3)
    B, H, L, D = q.shape
    if tuple(k.shape) != (B, L, D) or tuple(v.shape) != (B, L, D):
        raise ValueError("k and v must be [B,L,D] with q [B,H,L,D]")
    if _bias_stride(bias, B, H, L, block) != 0:
        raise ValueError("ag_attn_fwd_noalloc takes one bias shared by the batch")
    _check_out(out, lse, B, H, L, D)
    with torch.cuda.device(_one_device(q, k, v, bias, out, lse)):
        st = lib.ag_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                     bias.data_ptr(), B, H, L, D, int(block),
                                     float(cap), out.data_ptr(), lse.data_ptr(),
                                     _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_attn_fwd_noalloc", st)
    return out, lse


def ag_attn_fwd_launch_count(B: int, L: int, cap: float = 5.0, H: int = 8,
                             D: int = 128, block: int = 16) -> int:
    """How many kernels ag_attn_fwd launches for these sizes (see include/ag.h)."""
    n = ctypes.c_int(-1)
    st = lib.ag_attn_fwd_launch_count(int(B), int(H), int(L), int(D), int(block),
                                      float(cap), ctypes.byref(n))
    if st != AG_OK:
        raise AgError("ag_attn_fwd_launch_count", st)
    return int(n.value)


def ag_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bias: torch.Tensor,
                lse: torch.Tensor, dout: torch.Tensor, cap: float = 5.0, block: int = 16,
                stream=None):
    """Backward of ag_attn_fwd (libag kernels): gradients of out for the
    upstream gradient dout [B,H,L,Dv] fp32, given the forward's lse.
    Returns (dq [B,H,L,D], dk [B,L,D], dv [B,L,Dv], dbias (bias's shape; a
    shared [H,P,P] bias gets the sum over the batch), delta [B,H,L]), all
    fp32 and newly allocated."""
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check(lse, "lse", torch.float32, 3)
    _check(dout, "dout", torch.float32, 4)
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    if tuple(k.shape) != (B, L, D) or tuple(v.shape) != (B, L, Dv):
        raise ValueError("k must be [B,L,D] and v [B,L,Dv] with q [B,H,L,D]")
    if tuple(lse.shape) != (B, H, L) or tuple(dout.shape) != (B, H, L, Dv):
        raise ValueError("lse must be [B,H,L] and dout [B,H,L,Dv]")
    bstride = _bias_stride(bias, B, H, L, block)
    dev = _one_device(q, k, v, bias, lse, dout)
    f32 = dict(dtype=torch.float32, device=dev)
    dq = torch.empty((B, H, L, D), **f32)
    dk = torch.empty((B, L, D), **f32)
    dv = torch.empty((B, L, Dv), **f32)
    dbias = torch.empty(tuple(bias.shape), **f32)
    delta = torch.empty((B, H, L), **f32)
    with torch.cuda.device(dev):
        st = lib.ag_attn_bwd(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), bias.data_ptr(), bstride,
            lse.data_ptr(), dout.data_ptr(), B, H, L, D, Dv, int(block), float(cap),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dbias.data_ptr(),
            delta.data_ptr(), _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_attn_bwd", st)
    return dq, dk, dv, dbias, delta


def ag_attn_bwd_launch_count(Dv: int = 128) -> int:
    """How many kernels a non-empty ag_attn_bwd call with value width Dv launches."""
    n = ctypes.c_int(-1)
    st = lib.ag_attn_bwd_launch_count(int(Dv), ctypes.byref(n))
    if st != AG_OK:
        raise AgError("ag_attn_bwd_launch_count", st)
    return int(n.value)


def ag_device_error(device: int = 0, clear: bool = True) -> int:
    """Synchronise `device` and return (and optionally clear) its error word."""
    code = ctypes.c_int(0)
    st = lib.ag_device_error(int(device), ctypes.byref(code), 1 if clear else 0)
    if st not in (AG_OK, 8):
        raise AgError("ag_device_error", st)
    return int(code.value)


def ag_debug_wait_timeout(timeout_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see include/ag.h)."""
    st = lib.ag_debug_wait_timeout(int(timeout_ns), _stream_ptr(stream))
    if st != AG_OK:
        raise AgError("ag_debug_wait_timeout", st)


INF = math.inf
