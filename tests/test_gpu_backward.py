"""bra_attend_backward (dQ, dK, dV for a fixed routing) against the float64
oracle's gradients, through the C ABI.

Tolerance.  The kernel reads exactly the values the oracle is given (bf16
inputs widened), so the only differences are fp32 rounding: dot products of
32 terms, softmax sums over at most 256 keys, dK/dV sums over the queries of
every region routing to a key (fp32 atomics, in any order).  The test allows
|err| <= 2e-4 * (1 + |ref|)."""
import numpy as np
import pytest

import bra_inputs as bi
import oracle
from gpu_helpers import device_inputs

pytestmark = pytest.mark.gpu


def run(shape: bi.BraShape, seed: int, idx=None):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    inp = bi.make_inputs(shape, seed)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    if idx is None:
        idx_d = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device="cuda")
        bra.bra_route(s, q, k, idx_d, ws)
    else:
        idx_d = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    rng = np.random.default_rng(seed + 100)
    go = torch.from_numpy(rng.standard_normal(q.shape).astype(np.float32)).to(q.dtype).cuda()
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device="cuda") for _ in range(3))
    bra.bra_attend_backward(s, q, k, v, idx_d, go, dq, dk, dv, ws)
    status = bra.bra_device_status(s, ws)
    torch.cuda.synchronize()
    ref = oracle.attention_backward(inp.q_f64, inp.k_f64, inp.v_f64, idx_d.cpu().numpy(),
                                    go.double().cpu().numpy(), shape.heads, shape.S) if status == bra.BRA_OK else None
    return status, (dq, dk, dv), ref


@pytest.mark.parametrize("name,shape", [
    ("tiny", bi.BraShape(1, 16, 16, 32, 1, 4, 2, "f32")),
    ("stage1_b4", bi.BraShape(4, 56, 56, 64, 2, 7, 1, "bf16")),
    ("stage2_b4", bi.BraShape(4, 28, 28, 128, 4, 7, 4, "bf16")),
    ("stage3_b4", bi.BraShape(4, 14, 14, 256, 8, 7, 16, "bf16")),
    ("dense_topk", bi.BraShape(1, 16, 16, 64, 2, 4, 16, "bf16")),
    ("ragged", bi.BraShape(2, 24, 24, 64, 2, 4, 3, "f32")),
])
def test_gradients_match_oracle(name, shape):
    import dynamic_sparse_attention_bra_b200 as bra
    status, got, ref = run(shape, 7)
    assert status == bra.BRA_OK
    for g_name, a, b in zip("qkv", got, ref):
        err = np.abs(a.double().cpu().numpy() - b)
        assert (err <= 2e-4 * (1 + np.abs(b))).all(), f"d{g_name}: max err {err.max():.3e}"


def test_repeated_routes_count_once():
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(1, 16, 16, 64, 2, 4, 3, "bf16")
    rng = np.random.default_rng(3)
    idx = rng.integers(0, shape.R, size=(shape.B, shape.heads, shape.R, shape.topk)).astype(np.int32)
    idx[..., 1] = idx[..., 0]  # every row lists a region twice
    status, got, ref = run(shape, 9, idx)
    assert status == bra.BRA_OK
    for a, b in zip(got, ref):
        err = np.abs(a.double().cpu().numpy() - b)
        assert (err <= 2e-4 * (1 + np.abs(b))).all(), err.max()


def test_out_of_range_route_is_reported():
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(1, 16, 16, 64, 2, 4, 2, "bf16")
    idx = np.zeros((shape.B, shape.heads, shape.R, shape.topk), dtype=np.int32)
    idx[0, 1, 3, 1] = shape.R + 5
    status, _, _ = run(shape, 11, idx)
    assert status == bra.BRA_ERR_BAD_ROUTE
