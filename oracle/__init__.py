"""Float64 CPU oracle for pair-bias multi-query attention (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference leg of ``bench.py`` are the only callers.  The
product package never imports this module and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, float64, OpenMP).  This
wrapper only converts inputs to contiguous float64 numpy arrays and calls it.
The definition it follows is Eq. L_ij of the page "Making Full-Context
AlphaGenome Fit on an RTX 3090" (section "Why stock FlashAttention was not a
drop-in replacement"), with the softmax over all keys and natural-log lse.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

_c_double_p = ctypes.POINTER(ctypes.c_double)
_c_int64_p = ctypes.POINTER(ctypes.c_int64)


def _f64(x) -> np.ndarray:
    """Exact widening of a torch tensor (bf16 / fp32 / fp64) or array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_c_double_p)


class Oracle:
    """Handle on one build of the oracle library (the default or a mutant)."""

    def __init__(self, libpath: str | None = None):
        if libpath is None:
            libpath = _build.ensure_built()
        self.libpath = libpath
        lib = ctypes.CDLL(libpath)
        L = ctypes.c_long
        lib.agref_pair_bias_project.argtypes = [
            _c_double_p, _c_double_p, _c_double_p, L, L, L, ctypes.c_int]
        lib.agref_attn_fwd_ex.argtypes = [
            _c_double_p, _c_double_p, _c_double_p, _c_double_p, L,
            L, L, L, L, L, L, ctypes.c_double,
            _c_double_p, _c_double_p, _c_double_p, ctypes.c_int]
        lib.agref_attn_rows_ex.argtypes = [
            _c_double_p, _c_double_p, _c_double_p, _c_double_p, L,
            L, L, L, L, L, L, ctypes.c_double,
            _c_int64_p, L, _c_double_p, _c_double_p, ctypes.c_int]
        lib.agref_attn_bwd_ex.argtypes = [
            _c_double_p, _c_double_p, _c_double_p, _c_double_p, L, _c_double_p,
            L, L, L, L, L, L, ctypes.c_double,
            _c_double_p, _c_double_p, _c_double_p, _c_double_p, _c_double_p,
            _c_double_p, ctypes.c_int]
        lib.agref_attn_bwd_sample.argtypes = [
            _c_double_p, _c_double_p, _c_double_p, _c_double_p, L, _c_double_p,
            L, L, L, L, L, L, ctypes.c_double,
            _c_int64_p, L, _c_double_p, _c_int64_p, L, _c_double_p, _c_double_p,
            _c_int64_p, L, _c_double_p, ctypes.c_int]
        lib.agref_max_threads.argtypes = [ctypes.c_int]
        for f in ("agref_pair_bias_project", "agref_attn_fwd_ex",
                  "agref_attn_rows_ex", "agref_attn_bwd_ex", "agref_attn_bwd_sample",
                  "agref_max_threads", "agref_mutant_id"):
            getattr(lib, f).restype = ctypes.c_int
        self._lib = lib
        self.mutant = lib.agref_mutant_id()

    def threads(self, nthreads: int = 0) -> int:
        """Set (if > 0) and return the OpenMP thread count the oracle uses."""
        return int(self._lib.agref_max_threads(int(nthreads)))

    # -- pair-bias projection -------------------------------------------------
    def pair_bias_project(self, pair, W, nthreads: int = 0) -> np.ndarray:
        """bias[h,p,q] = sum_c pair[p,q,c] * W[c,h]; pair [P,P,Cp], W [Cp,H]."""
        pair = _f64(pair)
        W = _f64(W)
        P, P2, Cp = pair.shape
        assert P == P2 and W.shape[0] == Cp
        H = W.shape[1]
        bias = np.empty((H, P, P), dtype=np.float64)
        rc = self._lib.agref_pair_bias_project(
            _ptr(pair), _ptr(W), _ptr(bias), P, Cp, H, int(nthreads))
        if rc != 0:
            raise ValueError(f"agref_pair_bias_project rc={rc}")
        return bias

    # -- attention ------------------------------------------------------------
    @staticmethod
    def _bias_stride(bias, B, H, L, block) -> int:
        """bias is [H,P,P] (shared by the batch) or [B,H,P,P] (one per item),
        P = ceil(L / block); returns the batch stride in doubles."""
        P = -(-L // block) if block > 0 else 0
        if bias.ndim == 3 and bias.shape == (H, P, P):
            return 0
        if bias.ndim == 4 and bias.shape == (B, H, P, P):
            return H * P * P
        raise ValueError(f"bias shape {bias.shape} is neither ({H},{P},{P}) "
                         f"nor ({B},{H},{P},{P})")

    def attn_fwd(self, q, k, v, bias, block: int = 16, cap: float = 5.0,
                 probs: bool = False, nthreads: int = 0):
        """Full attention: returns (out [B,H,L,Dv], lse [B,H,L]) and, if
        probs=True, also the softmax weights [B,H,L,L] (tiny inputs only).
        bias: [H,P,P] shared, or [B,H,P,P] per batch item; P = ceil(L/block)."""
        q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
        B, H, L, D = q.shape
        Dv = v.shape[-1]
        assert k.shape == (B, L, D) and v.shape == (B, L, Dv)
        bstride = self._bias_stride(bias, B, H, L, int(block))
        out = np.empty((B, H, L, Dv), dtype=np.float64)
        lse = np.empty((B, H, L), dtype=np.float64)
        pr = np.empty((B, H, L, L), dtype=np.float64) if probs else None
        rc = self._lib.agref_attn_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(bias), bstride, B, H, L, D, Dv, int(block),
            float(cap), _ptr(out), _ptr(lse),
            _ptr(pr) if probs else None, int(nthreads))
        if rc != 0:
            raise ValueError(f"agref_attn_fwd rc={rc}")
        return (out, lse, pr) if probs else (out, lse)

    def attn_rows(self, q, k, v, bias, rows, block: int = 16,
                  cap: float = 5.0, nthreads: int = 0):
        """Selected rows: rows is an int array [n,3] of (b, h, i).  Returns
        (out_rows [n,Dv], lse_rows [n])."""
        q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
        B, H, L, D = q.shape
        Dv = v.shape[-1]
        bstride = self._bias_stride(bias, B, H, L, int(block))
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows.shape[0]
        out = np.empty((n, Dv), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
        rc = self._lib.agref_attn_rows_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(bias), bstride, B, H, L, D, Dv, int(block),
            float(cap), rows.ctypes.data_as(_c_int64_p), n, _ptr(out),
            _ptr(lse), int(nthreads))
        if rc != 0:
            raise ValueError(f"agref_attn_rows rc={rc}")
        return out, lse

    # -- attention backward ---------------------------------------------------
    def attn_bwd(self, q, k, v, bias, dout, block: int = 16, cap: float = 5.0,
                 nthreads: int = 0):
        """Gradients of out for the upstream gradient dout [B,H,L,Dv]: returns
        (dq [B,H,L,D], dk [B,L,D], dv [B,L,Dv], dbias (bias's shape; a shared
        [H,P,P] bias gets the sum over the batch), lse [B,H,L], delta [B,H,L])
        with delta_i = sum_j p_ij * (dout_i . v_j)."""
        q, k, v, bias, dout = _f64(q), _f64(k), _f64(v), _f64(bias), _f64(dout)
        B, H, L, D = q.shape
        Dv = v.shape[-1]
        assert k.shape == (B, L, D) and v.shape == (B, L, Dv)
        assert dout.shape == (B, H, L, Dv)
        bstride = self._bias_stride(bias, B, H, L, int(block))
        dq = np.zeros((B, H, L, D))
        dk = np.zeros((B, L, D))
        dv = np.zeros((B, L, Dv))
        dbias = np.zeros(bias.shape)
        lse = np.zeros((B, H, L))
        delta = np.zeros((B, H, L))
        rc = self._lib.agref_attn_bwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(bias), bstride, _ptr(dout),
            B, H, L, D, Dv, int(block), float(cap), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(dbias), _ptr(lse), _ptr(delta), int(nthreads))
        if rc != 0:
            raise ValueError(f"agref_attn_bwd_ex rc={rc}")
        return dq, dk, dv, dbias, lse, delta

    def attn_bwd_sample(self, q, k, v, bias, dout, rows=(), keys=(), cells=(),
                        block: int = 16, cap: float = 5.0, nthreads: int = 0):
        """Selected gradients: rows (b,h,i) -> dq rows [n,D]; keys (b,j) ->
        dk rows [n,D] and dv rows [n,Dv]; cells (b,h,I,J) -> dbias values [n]
        (b ignored for a shared bias)."""
        q, k, v, bias, dout = _f64(q), _f64(k), _f64(v), _f64(bias), _f64(dout)
        B, H, L, D = q.shape
        Dv = v.shape[-1]
        bstride = self._bias_stride(bias, B, H, L, int(block))
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64).reshape(-1, 2))
        cells = np.ascontiguousarray(np.asarray(cells, dtype=np.int64).reshape(-1, 4))
        dq = np.zeros((rows.shape[0], D))
        dk = np.zeros((keys.shape[0], D))
        dv = np.zeros((keys.shape[0], Dv))
        db = np.zeros((cells.shape[0],))
        rc = self._lib.agref_attn_bwd_sample(
            _ptr(q), _ptr(k), _ptr(v), _ptr(bias), bstride, _ptr(dout),
            B, H, L, D, Dv, int(block), float(cap),
            rows.ctypes.data_as(_c_int64_p), rows.shape[0], _ptr(dq),
            keys.ctypes.data_as(_c_int64_p), keys.shape[0], _ptr(dk), _ptr(dv),
            cells.ctypes.data_as(_c_int64_p), cells.shape[0], _ptr(db), int(nthreads))
        if rc != 0:
            raise ValueError(f"agref_attn_bwd_sample rc={rc}")
        return dq, dk, dv, db


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from the unmodified source."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


INF = math.inf
