"""Guard bands around every output buffer: each kernel must write inside its
output and nowhere next to it.

Every output tensor is carved out of a larger buffer whose leading and
trailing bands (4 KiB each) hold a fixed byte pattern; after the call the
bands must be unchanged and the output must still match the oracle.  This is
the run-time check that stands in for a memory sanitizer (which this pool
does not offer): a kernel that writes one row past its output, or before it,
changes a band.
"""
import numpy as np
import pytest

import bra_inputs as bi
import oracle
from gpu_helpers import device_inputs
from parity import TOL

pytestmark = pytest.mark.gpu

BAND = 4096  # bytes on each side
PATTERN = 0xA5


def guarded(shape, dtype):
    """(buffer, view): a uint8 buffer with bands around a tensor of ``shape``."""
    import torch
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    buf = torch.full((BAND + n + BAND,), PATTERN, dtype=torch.uint8, device="cuda")
    view = buf[BAND:BAND + n].view(dtype).view(shape)
    return buf, view


def bands_intact(buf) -> bool:
    import torch
    torch.cuda.synchronize()
    head, tail = buf[:BAND], buf[-BAND:]
    return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


KERNEL_SHAPES = [
    ("slice", (2, 14, 14, 256, 8, 7, 16)),
    ("warp", (2, 28, 28, 128, 4, 7, 4)),
    ("flash", (1, 64, 64, 64, 2, 4, 2)),
    ("stack", (2, 56, 56, 64, 2, 7, 1)),
    ("tiled", (1, 32, 32, 64, 2, 2, 2)),
    ("simt", (1, 16, 16, 64, 2, 4, 3)),
]


@pytest.mark.parametrize("kernel,dims", KERNEL_SHAPES, ids=[k for k, _ in KERNEL_SHAPES])
def test_attention_writes_only_its_output(kernel, dims, monkeypatch):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    monkeypatch.setenv("BRA_ATTEND_KERNEL", kernel)
    B, H, W, C, heads, S, topk = dims
    shape = bi.BraShape(B, H, W, C, heads, S, topk, "bf16")
    inp = bi.make_inputs(shape, 61)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(B, H, W, C, heads, S, topk, "bf16")
    ws_buf, ws = guarded((bra.bra_workspace_bytes(s),), torch.uint8)
    ws.zero_()
    o_buf, o = guarded(tuple(q.shape), torch.bfloat16)
    i_buf, idx = guarded((B, heads, S * S, topk), torch.int32)
    bra.bra_forward(s, q, k, v, o, idx, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    assert bands_intact(o_buf) and bands_intact(i_buf) and bands_intact(ws_buf)
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx.cpu().numpy(), heads, S)
    assert np.abs(o.float().cpu().numpy() - ref).max() <= TOL["bf16"]


def test_projection_writes_only_its_outputs():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(2, 56, 56, 64, 2, 7, 1, "bf16")
    proj = bi.make_projection_inputs(shape, 62)
    x = torch.from_numpy(proj.x_store).view(torch.bfloat16).cuda()
    w = torch.from_numpy(proj.w_store).view(torch.bfloat16).cuda()
    b = torch.from_numpy(proj.b_store).cuda()
    s = bra.shape_for(*[getattr(shape, f) for f in "B H W C heads S topk".split()], "bf16")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    outs = [guarded(tuple(x.shape), torch.bfloat16) for _ in range(3)]
    means = [guarded((shape.B, shape.heads, shape.R, shape.d), torch.float32) for _ in range(2)]
    bra.bra_qkv_project(s, x, w, b, *[v for _, v in outs], *[v for _, v in means], ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    assert all(bands_intact(buf) for buf, _ in outs + means)


def test_local_context_writes_only_its_output():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    B, H, W, C = 2, 56, 56, 64
    rng = np.random.default_rng(63)
    v = torch.from_numpy(rng.standard_normal((B, H, W, C)).astype(np.float32)).to(torch.bfloat16).cuda()
    wt = torch.from_numpy((rng.standard_normal((C, 5, 5)) / 5).astype(np.float32)).cuda()
    o_buf, o = guarded((B, H, W, C), torch.bfloat16)
    o.zero_()
    s = bra.shape_for(B, H, W, C, 2, 1, 1, "bf16")
    bra.bra_lce(s, v, wt, None, o)
    assert bands_intact(o_buf)


def test_forward_lce_writes_only_its_outputs():
    """bra_forward_lce (the local context term in the attention epilogue)."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(2, 56, 56, 64, 2, 7, 1, "bf16")
    inp = bi.make_inputs(shape, 65)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(*[getattr(shape, f) for f in "B H W C heads S topk".split()], "bf16")
    ws_buf, ws = guarded((bra.bra_workspace_bytes(s),), torch.uint8)
    ws.zero_()
    rng = np.random.default_rng(66)
    wt = torch.from_numpy((rng.standard_normal((shape.C, 5, 5)) / 5).astype(np.float32)).cuda()
    bias = torch.from_numpy(rng.standard_normal(shape.C).astype(np.float32)).cuda()
    o_buf, o = guarded(tuple(q.shape), torch.bfloat16)
    idx_buf, idx = guarded((shape.B, shape.heads, shape.R, shape.topk), torch.int32)
    bra.bra_forward_lce(s, q, k, v, wt, bias, o, idx, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    assert all(bands_intact(buf) for buf in (o_buf, idx_buf, ws_buf))


@pytest.mark.parametrize("kernel,dims", [("mma", (2, 56, 56, 64, 2, 7, 1)), ("mma", (2, 28, 28, 128, 4, 7, 4)),
                                         ("simt", (2, 56, 56, 64, 2, 7, 1))],
                         ids=["mma_stage1", "mma_stage2", "simt_stage1"])
def test_backward_writes_only_its_outputs(kernel, dims, monkeypatch):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    monkeypatch.setenv("BRA_BACKWARD_KERNEL", kernel)
    shape = bi.BraShape(*dims, "bf16")
    inp = bi.make_inputs(shape, 64)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(*[getattr(shape, f) for f in "B H W C heads S topk".split()], "bf16")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device="cuda")
    bra.bra_route(s, q, k, idx, ws)
    go = torch.randn(q.shape, device="cuda").to(torch.bfloat16)
    grads = [guarded(tuple(q.shape), torch.float32) for _ in range(3)]
    bra.bra_attend_backward(s, q, k, v, idx, go, *[g for _, g in grads], ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    assert all(bands_intact(buf) for buf, _ in grads)
