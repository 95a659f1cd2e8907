"""Float64 CPU oracle for Bi-Level Routing Attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it; the library's product path never does.
It shares no code with the CUDA path (see ``bra_oracle.c`` for the method's
steps and the readings taken where the pages are silent).

Every function here is a thin ctypes wrapper over ``bra_oracle.c``; inputs
are converted to contiguous float64, outputs are returned as new arrays.

Parity status: the 1/sqrt(d) logit scale, per-head routing and row-major
token order are readings of the pages, not values the pages fix, so those
three choices are "parity unpinned"; every other step is pinned by the
tests in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bra_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_bra.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_i = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile ``bra_oracle.c`` into ``liboracle_bra.so`` (plain gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_region_pool.argtypes = [_dp, _i, _i, _i, _i, _i, _i, _dp]
    lib.oracle_region_affinity.argtypes = [_dp, _dp, _i, _i, _i, _i, _dp]
    lib.oracle_topk_routing.argtypes = [_dp, _i, _i, _i, _i, _ip]
    lib.oracle_token_attention.argtypes = [_dp, _dp, _dp, _i, _i, _i, _i, _i, _i, _i, _ip, _dp]
    lib.oracle_bra_forward.argtypes = [_dp, _dp, _dp, _i, _i, _i, _i, _i, _i, _i, _dp, _ip, _dp]
    lib.oracle_local_context.argtypes = [_dp, _i, _i, _i, _i, _dp, _dp, _dp]
    lib.oracle_attention_backward.argtypes = [_dp, _dp, _dp, _i, _i, _i, _i, _i, _i, _i, _ip, _dp, _dp, _dp, _dp]
    lib.oracle_qkv_projection.argtypes = [_dp, _i, _i, _i, _i, _dp, _dp, _dp, _dp, _dp]
    for f in (lib.oracle_region_pool, lib.oracle_region_affinity, lib.oracle_topk_routing,
              lib.oracle_token_attention, lib.oracle_bra_forward):
        f.restype = _i
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


@contextlib.contextmanager
def swapped_library(path: str):
    """Run the wrappers against another build of ``bra_oracle.c`` (the tests
    use it to check that deliberately broken oracles fail the pins)."""
    global _lib
    saved = _load()
    _lib = _bind(path)
    try:
        yield
    finally:
        _lib = saved


def _f64(x) -> np.ndarray:
    """Contiguous float64 copy of an input; NaN and infinity are outside the
    method's contract (the pages define the steps on real-valued maps), so they
    are rejected rather than propagated."""
    a = np.ascontiguousarray(x, dtype=np.float64)
    if not np.isfinite(a).all():
        raise ValueError("oracle inputs must be finite (NaN and infinity are outside the contract)")
    return a


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def region_pool(x, heads: int, S: int) -> np.ndarray:
    """Per-region mean of map ``x`` [B,H,W,C] -> [B, heads, S*S, d]."""
    x = _f64(x)
    B, H, W, C = x.shape
    out = np.zeros((B, heads, S * S, C // heads if heads else 0), dtype=np.float64)
    _check(_load().oracle_region_pool(_ptr(x, _dp), B, H, W, C, heads, S, _ptr(out, _dp)), "pool")
    return out


def region_affinity(qr, kr) -> np.ndarray:
    """A^r = Q^r (K^r)^T per (batch, head): [B,heads,R,d] x2 -> [B,heads,R,R]."""
    qr, kr = _f64(qr), _f64(kr)
    B, heads, R, d = qr.shape
    out = np.zeros((B, heads, R, R), dtype=np.float64)
    _check(_load().oracle_region_affinity(_ptr(qr, _dp), _ptr(kr, _dp), B, heads, R, d,
                                          _ptr(out, _dp)), "affinity")
    return out


def topk_routing(a, topk: int) -> np.ndarray:
    """I^r: per row, the topk regions by (affinity desc, index asc) -> int32."""
    a = _f64(a)
    B, heads, R, _ = a.shape
    out = np.zeros((B, heads, R, topk), dtype=np.int32)
    _check(_load().oracle_topk_routing(_ptr(a, _dp), B, heads, R, topk, _ptr(out, _ip)), "topk")
    return out


def token_attention(q, k, v, idx, heads: int, S: int) -> np.ndarray:
    """Token-to-token attention of every query over its routed regions' tokens."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    B, H, W, C = q.shape
    topk = idx.shape[-1]
    out = np.zeros_like(q)
    _check(_load().oracle_token_attention(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, H, W, C,
                                          heads, S, topk, _ptr(idx, _ip), _ptr(out, _dp)),
           "attention")
    return out


def bra_forward(q, k, v, heads: int, S: int, topk: int, want_affinity: bool = False):
    """All steps: returns (O, I^r) or (O, I^r, A^r)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, W, C = q.shape
    R = S * S
    o = np.zeros_like(q)
    idx = np.zeros((B, heads, R, topk), dtype=np.int32)
    a = np.zeros((B, heads, R, R), dtype=np.float64) if want_affinity else None
    rc = _load().oracle_bra_forward(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, H, W, C, heads,
                                    S, topk, _ptr(o, _dp), _ptr(idx, _ip),
                                    _ptr(a, _dp) if a is not None else None)
    _check(rc, "forward")
    return (o, idx, a) if want_affinity else (o, idx)


def local_context(v, weight, bias=None) -> np.ndarray:
    """5x5 depthwise filter of V (zero padding 2, cross-correlation) plus bias:
    the local context enhancement term added to the attention output.
    ``weight`` is [C, 5, 5] (a [C, 1, 5, 5] layer weight reshaped), ``bias`` [C]
    or None."""
    v = _f64(v)
    B, H, W, C = v.shape
    w = _f64(np.reshape(weight, (C, 5, 5)))
    bb = _f64(bias) if bias is not None else None
    out = np.zeros_like(v)
    _check(_load().oracle_local_context(_ptr(v, _dp), B, H, W, C, _ptr(w, _dp),
                                        _ptr(bb, _dp) if bb is not None else None, _ptr(out, _dp)),
           "local context")
    return out


def attention_backward(q, k, v, idx, grad_o, heads: int, S: int):
    """Gradients (dQ, dK, dV) of the token attention for a fixed routing
    ``idx`` and an incoming gradient ``grad_o`` of O; a region repeated in a
    routing row counts once."""
    q, k, v, gr = _f64(q), _f64(k), _f64(v), _f64(grad_o)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    B, H, W, C = q.shape
    topk = idx.shape[-1]
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    _check(_load().oracle_attention_backward(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, H, W, C, heads, S, topk,
                                             _ptr(idx, _ip), _ptr(gr, _dp), _ptr(dq, _dp), _ptr(dk, _dp),
                                             _ptr(dv, _dp)),
           "attention backward")
    return dq, dk, dv


def qkv_projection(x, weight, bias=None):
    """Q, K, V of a feature map X [B, H, W, C]: the three channel chunks of
    the linear layer ``x @ weight.T + bias`` with ``weight`` [3C, C] and
    ``bias`` [3C] or None."""
    x = _f64(x)
    B, H, W, C = x.shape
    w = _f64(np.reshape(weight, (3 * C, C)))
    bb = _f64(np.reshape(bias, (3 * C,))) if bias is not None else None
    q, k, v = np.zeros_like(x), np.zeros_like(x), np.zeros_like(x)
    _check(_load().oracle_qkv_projection(_ptr(x, _dp), B, H, W, C, _ptr(w, _dp),
                                         _ptr(bb, _dp) if bb is not None else None,
                                         _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp)),
           "qkv projection")
    return q, k, v
