"""bra_route_noalloc: routing for callers that cannot allocate device memory
(for example a plugin inside a framework that owns all GPU memory and gives
it no workspace, or a loop where cudaMalloc's device-wide synchronisation is
not allowed).  Its scratch is a fixed array inside the library.

The GPU test compares it with bra_route (which uses a caller workspace) on
two calls in a row with different workloads, so the array's leftover
contents from the first call must not matter to the second.  This file is
collected last on purpose.
"""
import ctypes

import pytest
import torch

import bra_inputs as bi
import dynamic_sparse_attention_bra_b200 as bra
from gpu_helpers import device_inputs


def routes_both_ways(name):
    shape, seed = bi.WORKLOADS[name]
    q, k, _ = device_inputs(bi.make_inputs(shape, seed))
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    dims = (shape.B, shape.heads, shape.R, shape.topk)
    ref = torch.full(dims, -7, dtype=torch.int32, device="cuda")
    got = torch.full(dims, -7, dtype=torch.int32, device="cuda")
    bra.bra_route(s, q, k, ref, ws)
    bra.bra_route_noalloc(s, q, k, got)
    torch.cuda.synchronize()
    return ref, got


@pytest.mark.gpu
def test_noalloc_matches_workspace_route_twice():
    for name in ("stage3", "stage2"):  # largest means first, then a smaller problem
        ref, got = routes_both_ways(name)
        assert torch.equal(ref, got), name  # routing indices: bit-exact


def test_noalloc_rejects_oversize_before_launch():
    # B * heads * R * d = 128 * 8 * 49 * 32 > BRA_NOALLOC_MAX_MEANS: refused on the host
    s = bra.shape_for(128, 14, 14, 256, 8, 7, 16, "bf16")
    assert 128 * 8 * 49 * 32 > bra.NOALLOC_MAX_MEANS
    p = 1 << 20
    assert bra._lib.bra_route_noalloc(ctypes.byref(s), p, p, p, None) == bra.BRA_ERR_UNSUPPORTED
    bad = bra.shape_for(1, 16, 16, 64, 2, 5, 1, "bf16")  # S does not divide 16
    assert bra._lib.bra_route_noalloc(ctypes.byref(bad), p, p, p, None) == bra.BRA_ERR_INVALID_ARG
    assert bra._lib.bra_route_noalloc(None, p, p, p, None) == bra.BRA_ERR_INVALID_ARG
