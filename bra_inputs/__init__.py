"""Seeded synthetic inputs for Bi-Level Routing Attention workloads.

This module is the only code shared by the CUDA path's tests/bench and the
float64 oracle.  It holds no arithmetic of the attention method itself: it
only draws region-correlated Gaussian feature maps and rounds them to the
storage type the GPU reads.

Recipe (one tensor X in {Q, K, V}, channels-last [B, H, W, C]):

    mu[b, r, c]   ~ N(0, 1)        one vector per (batch, region)
    eps[b, y, x, c] ~ N(0, 1)
    X[b, y, x, c] = mu[b, region(y, x), c] + 0.5 * eps[b, y, x, c]

where region(y, x) = (y // (H/S)) * S + (x // (W/S)) numbers the S x S grid
row-major.  The region structure mimics what a projected feature map of a
natural image looks like to the router: neighbouring tokens share content.

Random numbers come from a counter-based generator: splitmix64 (Steele,
Lea, Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014)
applied to ``key(seed, stream) + (i + 1) * 0x9E3779B97F4A7C15`` for element
counter ``i``, turned into doubles in (0, 1) with 53 random bits and into
normals with the Box-Muller transform (pairs (2j, 2j+1) give cos/sin).
Streams: Q = 0, K = 1, V = 2; means and noise use sub-streams 0 and 1.

Projection workloads (the Q, K, V linear layer in front of the path) draw
the feature map X with the same recipe on stream 3, and the layer's
parameters the way a freshly initialised linear layer holds them:
W [3C, C] and b [3C] uniform in (-1/sqrt(C), 1/sqrt(C)), from the uniform
streams 8 (W) and 9 (b).
"""
from __future__ import annotations

import dataclasses

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


_CHUNK = 1 << 20


def _mix(z: np.ndarray, t: np.ndarray) -> None:
    """splitmix64 finaliser, in place on uint64 ``z`` (``t`` is scratch)."""
    for shift, mul in ((30, _M1), (27, _M2)):
        np.right_shift(z, np.uint64(shift), out=t)
        np.bitwise_xor(z, t, out=z)
        np.multiply(z, mul, out=z)
    np.right_shift(z, np.uint64(31), out=t)
    np.bitwise_xor(z, t, out=z)


def _key(seed: int, stream: int) -> np.uint64:
    s = np.array([(seed * 0x100000001B3 + stream * 0x2545F4914F6CDD1D + 1) & 0xFFFFFFFFFFFFFFFF],
                 dtype=np.uint64)
    _mix(s, np.empty_like(s))
    return s[0]


def splitmix_u64(seed: int, stream: int, count: int) -> np.ndarray:
    """``count`` 64-bit words of the counter-based splitmix64 stream."""
    out = np.empty(count, dtype=np.uint64)
    key = _key(seed, stream)
    t = np.empty(min(count, _CHUNK), dtype=np.uint64)
    with np.errstate(over="ignore"):
        for lo in range(0, count, _CHUNK):
            z = out[lo:lo + _CHUNK]
            z[:] = np.arange(lo + 1, lo + 1 + z.size, dtype=np.uint64)
            np.multiply(z, _GOLDEN, out=z)
            np.add(z, key, out=z)
            _mix(z, t[:z.size])
    return out


def uniform01(seed: int, stream: int, count: int) -> np.ndarray:
    """Doubles strictly inside (0, 1): (top 53 bits + 0.5) * 2^-53."""
    w = splitmix_u64(seed, stream, count)
    np.right_shift(w, np.uint64(11), out=w)
    u = w.view(np.float64)  # reuse the buffer: int -> float conversion in place, by chunks
    for lo in range(0, count, _CHUNK):
        u[lo:lo + _CHUNK] = w[lo:lo + _CHUNK].astype(np.float64)
    u += 0.5
    u *= 1.0 / 9007199254740992.0
    return u


def normal(seed: int, stream: int, count: int) -> np.ndarray:
    """Standard normals by Box-Muller over consecutive uniform pairs."""
    pairs = (count + 1) // 2
    u = uniform01(seed, stream, 2 * pairs).reshape(pairs, 2)
    for lo in range(0, pairs, _CHUNK):
        blk = u[lo:lo + _CHUNK]
        rad = np.sqrt(-2.0 * np.log(blk[:, 0]))
        ang = (2.0 * np.pi) * blk[:, 1]
        blk[:, 0] = rad * np.cos(ang)
        blk[:, 1] = rad * np.sin(ang)
    return u.reshape(-1)[:count]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as int16 (same bits as uint16).  Inputs are
    finite by construction, so no NaN handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).copy()
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    # finite float32 patterns stay below 2^32 after adding at most 0x8000
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= np.uint32(16)
    return u.astype(np.uint16).view(np.int16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (int16/uint16) to float64 exactly."""
    u = np.ascontiguousarray(b).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


@dataclasses.dataclass(frozen=True)
class BraShape:
    """Problem size of one BRA call: feature map [B, H, W, C], heads, S, topk."""
    B: int
    H: int
    W: int
    C: int
    heads: int
    S: int
    topk: int
    dtype: str  # "f32" or "bf16"

    @property
    def d(self) -> int:
        return self.C // self.heads

    @property
    def R(self) -> int:
        return self.S * self.S

    @property
    def n(self) -> int:
        return (self.H // self.S) * (self.W // self.S)

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.W


# The five workload shapes: a tiny fp32 case, the three BiFormer stages at
# 224x224 input with S = 7 and topk = 1, 4, 16 (stage channels 64/128/256,
# head dim 32), and a dense-prediction map with S = 8.
WORKLOADS = {
    "tiny": (BraShape(1, 16, 16, 32, 1, 4, 2, "f32"), 0),
    "stage1": (BraShape(64, 56, 56, 64, 2, 7, 1, "bf16"), 1),
    "stage2": (BraShape(64, 28, 28, 128, 4, 7, 4, "bf16"), 2),
    "stage3": (BraShape(64, 14, 14, 256, 8, 7, 16, "bf16"), 3),
    "highres": (BraShape(2, 128, 128, 64, 2, 8, 4, "bf16"), 4),
    # object detection uses S = 16 (a 512 x 512 input at stride 4: 128 x 128 tokens,
    # 256 regions of 8 x 8)
    "detection": (BraShape(2, 128, 128, 64, 2, 16, 4, "bf16"), 5),
}


def region_map(H: int, W: int, S: int) -> np.ndarray:
    """[H, W] array of row-major region numbers of the S x S grid."""
    hs, ws = H // S, W // S
    y = np.arange(H)[:, None] // hs
    x = np.arange(W)[None, :] // ws
    return (y * S + x).astype(np.int64)


def feature_map(shape: BraShape, seed: int, stream: int) -> np.ndarray:
    """One region-correlated Gaussian map [B, H, W, C] in float64."""
    B, H, W, C, R = shape.B, shape.H, shape.W, shape.C, shape.R
    mu = normal(seed, 2 * stream, B * R * C).reshape(B, R, C)
    x = normal(seed, 2 * stream + 1, B * H * W * C).reshape(B, H, W, C)
    reg = region_map(H, W, shape.S)
    x *= 0.5
    for b in range(B):
        x[b] += mu[b, reg, :]
    return x


class BraInputs:
    """Q, K, V as stored for the GPU (``*_store``: float32, or bfloat16 bit
    patterns as int16) and, on first use, exactly widened to float64
    (``*_f64``), which is what the oracle consumes."""

    def __init__(self, shape: BraShape, q_store, k_store, v_store):
        self.shape = shape
        self.q_store, self.k_store, self.v_store = q_store, k_store, v_store
        self._wide = {}

    def _widen(self, name: str) -> np.ndarray:
        if name not in self._wide:
            st = getattr(self, name + "_store")
            self._wide[name] = (st.astype(np.float64) if self.shape.dtype == "f32"
                                else bf16_bits_to_f64(st))
        return self._wide[name]

    q_f64 = property(lambda self: self._widen("q"))
    k_f64 = property(lambda self: self._widen("k"))
    v_f64 = property(lambda self: self._widen("v"))


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    f32 = x.astype(np.float32)
    if dtype == "f32":
        return f32
    if dtype == "bf16":
        return f32_to_bf16_bits(f32)
    raise ValueError(f"unknown dtype {dtype!r}")


def make_inputs(shape: BraShape, seed: int) -> BraInputs:
    """Q, K, V for ``shape``: generated in float64, rounded to float32, then
    (bf16 workloads) rounded to bfloat16."""
    stores = [_store(feature_map(shape, seed, stream), shape.dtype) for stream in (0, 1, 2)]
    return BraInputs(shape, *stores)


class ProjectionInputs:
    """X [B, H, W, C] and W [3C, C] as bfloat16 bit patterns (int16), b [3C]
    as float32, plus their exact float64 widenings for the oracle."""

    def __init__(self, shape: BraShape, x_store, w_store, b_store):
        self.shape = shape
        self.x_store, self.w_store, self.b_store = x_store, w_store, b_store
        self.x_f64 = bf16_bits_to_f64(x_store)
        self.w_f64 = bf16_bits_to_f64(w_store)
        self.b_f64 = b_store.astype(np.float64)


def make_projection_inputs(shape: BraShape, seed: int) -> ProjectionInputs:
    """Feature map and linear-layer parameters for the fused projection."""
    if shape.dtype != "bf16":
        raise ValueError("the projection workloads are bf16")
    C = shape.C
    bound = 1.0 / np.sqrt(C)
    x = _store(feature_map(shape, seed, 3), "bf16")
    w = _store(((2.0 * uniform01(seed, 8, 3 * C * C) - 1.0) * bound).reshape(3 * C, C), "bf16")
    b = ((2.0 * uniform01(seed, 9, 3 * C) - 1.0) * bound).astype(np.float32)
    return ProjectionInputs(shape, x, w, b)
