"""Bi-Level Routing Attention (BiFormer) forward on B200, sm_100a.

A thin ctypes binding over the C ABI of ``libbra_b200.so`` (declared in
``include/bra.h``).  Every step of the path runs in the library's CUDA
kernels; this module only turns torch tensors into pointers and sizes and
turns status codes into exceptions.  There is no CPU fallback: if the
library is missing the import of the binding fails.

Entry points (same names as the C ABI):

    bra_workspace_bytes(shape)
    bra_route(shape, q, k, idx, workspace, stream=None)
    bra_attend(shape, q, k, v, idx, o, workspace, stream=None)
    bra_forward(shape, q, k, v, o, idx, workspace, stream=None)
    bra_device_status(shape, workspace, stream=None)

and a convenience wrapper ``forward(q, k, v, heads, S, topk)`` that
allocates the outputs and workspace with torch and returns ``(o, idx)``.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "BraError", "BraShape", "shape_for", "bra_workspace_bytes", "bra_route", "bra_attend",
    "bra_forward", "bra_device_status", "bra_status_string", "forward", "library_path",
    "bra_route_noalloc", "bra_lce", "bra_selftest_bounded_wait", "bra_attend_backward",
    "bra_qkv_project", "bra_forward_qkv", "bra_forward_lce", "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
# BRA_LIBRARY selects another build of the same library, e.g. the debug build
# libbra_b200_debug.so (output-index checks in the attention kernels).
library_path = os.environ.get("BRA_LIBRARY") or os.path.join(_HERE, "libbra_b200.so")
debug_library_path = os.path.join(_HERE, "libbra_b200_debug.so")

(BRA_OK, BRA_ERR_INVALID_ARG, BRA_ERR_UNSUPPORTED, BRA_ERR_CUDA, BRA_ERR_TIMEOUT, BRA_ERR_BAD_ROUTE,
 BRA_ERR_BOUNDS) = range(7)
BRA_DTYPE_F32, BRA_DTYPE_BF16 = 0, 1

EXPORTED_SYMBOLS = ("bra_workspace_bytes", "bra_route", "bra_attend", "bra_forward",
                    "bra_device_status", "bra_status_string", "bra_version", "bra_route_noalloc",
                    "bra_lce", "bra_selftest_bounded_wait", "bra_attend_backward", "bra_qkv_project",
                    "bra_forward_qkv", "bra_forward_lce")
NOALLOC_MAX_MEANS = 1 << 20  # BRA_NOALLOC_MAX_MEANS


class BraShape(ctypes.Structure):
    """Mirror of ``bra_shape``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int), ("C", ctypes.c_int),
                ("heads", ctypes.c_int), ("S", ctypes.c_int), ("topk", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class BraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {bra_status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is not built; run `python dynamic_sparse_attention_bra_b200/build.py`")
    lib = ctypes.CDLL(library_path)
    vp, sp = ctypes.c_void_p, ctypes.POINTER(BraShape)
    lib.bra_workspace_bytes.argtypes = [sp]
    lib.bra_workspace_bytes.restype = ctypes.c_size_t
    lib.bra_route.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.bra_attend.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp]
    lib.bra_forward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp]
    lib.bra_lce.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.bra_forward_lce.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.bra_selftest_bounded_wait.argtypes = [sp, vp, ctypes.c_uint, ctypes.c_int, vp]
    lib.bra_attend_backward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.bra_qkv_project.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.bra_forward_qkv.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.bra_device_status.argtypes = [sp, vp, vp]
    lib.bra_route_noalloc.argtypes = [sp, vp, vp, vp, vp]
    lib.bra_route_noalloc.restype = ctypes.c_int
    for f in (lib.bra_route, lib.bra_attend, lib.bra_forward, lib.bra_device_status):
        f.restype = ctypes.c_int
    lib.bra_status_string.argtypes = [ctypes.c_int]
    lib.bra_status_string.restype = ctypes.c_char_p
    lib.bra_version.argtypes = []
    lib.bra_version.restype = ctypes.c_int
    return lib


_lib = _load()


def bra_status_string(status: int) -> str:
    return _lib.bra_status_string(status).decode()


def shape_for(B: int, H: int, W: int, C: int, heads: int, S: int, topk: int, dtype) -> BraShape:
    """``bra_shape`` for a problem; ``dtype`` is a torch dtype or "f32"/"bf16"."""
    name = str(dtype)
    code = BRA_DTYPE_BF16 if "bf16" in name or "bfloat16" in name else BRA_DTYPE_F32
    return BraShape(B, H, W, C, heads, S, topk, code)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(status: int, where: str):
    if status != BRA_OK:
        raise BraError(status, where)


def bra_workspace_bytes(shape: BraShape) -> int:
    return int(_lib.bra_workspace_bytes(ctypes.byref(shape)))


def bra_route(shape: BraShape, q, k, idx, workspace, stream=None) -> None:
    _check(_lib.bra_route(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(idx), _ptr(workspace),
                          _stream(stream)), "bra_route")


def bra_attend(shape: BraShape, q, k, v, idx, o, workspace, stream=None) -> None:
    _check(_lib.bra_attend(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o),
                           _ptr(workspace), _stream(stream)), "bra_attend")


def bra_forward(shape: BraShape, q, k, v, o, idx, workspace, stream=None) -> None:
    _check(_lib.bra_forward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(idx),
                            _ptr(workspace), _stream(stream)), "bra_forward")


def bra_attend_backward(shape: BraShape, q, k, v, idx, grad_o, dq, dk, dv, workspace, stream=None) -> None:
    """dQ, dK, dV (fp32 tensors, overwritten) of bra_attend for the fixed routing ``idx``."""
    _check(_lib.bra_attend_backward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(grad_o),
                                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), _stream(stream)),
           "bra_attend_backward")


def bra_qkv_project(shape: BraShape, x, w_qkv, b_qkv, q, k, v, q_r, k_r, workspace, stream=None) -> None:
    """[q | k | v] = x w_qkv^T (+ b_qkv) in bf16 and the fp32 region means q_r, k_r of q and k."""
    _check(_lib.bra_qkv_project(ctypes.byref(shape), _ptr(x), _ptr(w_qkv), _ptr(b_qkv) if b_qkv is not None else None,
                                _ptr(q), _ptr(k), _ptr(v), _ptr(q_r), _ptr(k_r), _ptr(workspace), _stream(stream)),
           "bra_qkv_project")


def bra_forward_qkv(shape: BraShape, x, w_qkv, b_qkv, q, k, v, o, idx, workspace, stream=None) -> None:
    """The path from the feature map x: projection with region means, routing, attention."""
    _check(_lib.bra_forward_qkv(ctypes.byref(shape), _ptr(x), _ptr(w_qkv), _ptr(b_qkv) if b_qkv is not None else None,
                                _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(idx), _ptr(workspace), _stream(stream)),
           "bra_forward_qkv")


def bra_selftest_bounded_wait(shape: BraShape, workspace, tries: int, arrive: bool, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see include/bra.h); read the
    outcome with bra_device_status."""
    _check(_lib.bra_selftest_bounded_wait(ctypes.byref(shape), _ptr(workspace), tries, 1 if arrive else 0,
                                          _stream(stream)), "bra_selftest_bounded_wait")


def bra_lce(shape: BraShape, v, weight, bias, o, stream=None) -> None:
    """o += bias + 5x5 depthwise filter of v (weight fp32 [C, 5, 5], bias fp32 [C] or None)."""
    _check(_lib.bra_lce(ctypes.byref(shape), _ptr(v), _ptr(weight), _ptr(bias) if bias is not None else None,
                        _ptr(o), _stream(stream)), "bra_lce")


def bra_forward_lce(shape: BraShape, q, k, v, weight, bias, o, idx, workspace, stream=None) -> None:
    """Routing, attention and the local context term (weight [C,5,5] fp32, bias [C] or None) in one call."""
    _check(_lib.bra_forward_lce(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(weight),
                                _ptr(bias) if bias is not None else None, _ptr(o), _ptr(idx), _ptr(workspace),
                                _stream(stream)), "bra_forward_lce")


def bra_route_noalloc(shape: BraShape, q, k, idx, stream=None) -> None:
    """bra_route with the library's own fixed scratch: for callers that cannot
    allocate device memory (see include/bra.h for the size limit and the
    rule that overlapping calls race)."""
    _check(_lib.bra_route_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(idx), _stream(stream)),
           "bra_route_noalloc")


def bra_device_status(shape: BraShape, workspace, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status code."""
    return int(_lib.bra_device_status(ctypes.byref(shape), _ptr(workspace), _stream(stream)))


def _check_tensor(t, name: str, dtype, numel: int):
    import torch
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous() and t.dtype == dtype
            and t.numel() == numel):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor of {numel} elements")


def forward(q, k, v, heads: int, S: int, topk: int, stream=None):
    """O, I^r for channels-last q, k, v [B, H, W, C] (float32 or bfloat16).

    Allocates O [B, H, W, C], I^r int32 [B, heads, S*S, topk] and a zeroed
    workspace with torch on q's device, then runs ``bra_forward``."""
    import torch
    B, H, W, C = q.shape
    shape = shape_for(B, H, W, C, heads, S, topk, q.dtype)
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, name, q.dtype, B * H * W * C)
    nbytes = bra_workspace_bytes(shape)
    if nbytes == 0:
        raise BraError(BRA_ERR_INVALID_ARG, "forward")
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    idx = torch.empty((B, heads, S * S, topk), dtype=torch.int32, device=q.device)
    bra_forward(shape, q, k, v, o, idx, ws, stream)
    return o, idx
