"""bra_forward_lce (routing, token attention and the local context term in
one call) against the float64 oracle, through the C ABI.

Routing is compared under the rule in ``parity.py``; O against
oracle.token_attention on the GPU's routing plus oracle.local_context on the
same V, weights and bias.  Tolerance (bf16): the attention's own bound
(2e-2, the bf16 P and the exponent rounding) plus one rounding of the sum to
bf16, at most half an ulp of the result, allowed as |ref| * 2^-8; the fp32
filter sum (25 products of O(1) values) adds about 1e-5.

The 8 x 8-region shapes with an even number of heads run the filter in the
attention kernel's epilogue (one kernel, O rounded once); the others run the
attention and then the filter (O rounded twice: the bound above also covers
the extra half ulp of the attention result).
"""
import numpy as np
import pytest

import bra_inputs as bi
import oracle
from gpu_helpers import device_inputs
from parity import TOL, compare_routes, record_margin

pytestmark = pytest.mark.gpu


def lce_params(C: int, seed: int, with_bias: bool = True):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((C, 5, 5)) / 5.0).astype(np.float32)
    b = rng.standard_normal(C).astype(np.float32) if with_bias else None
    return w, b


def check_forward_lce(shape: bi.BraShape, seed: int, label: str, with_bias: bool = True):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    inp = bi.make_inputs(shape, seed)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    w, b = lce_params(shape.C, seed + 1, with_bias)
    w_d = torch.from_numpy(w).cuda()
    b_d = torch.from_numpy(b).cuda() if b is not None else None
    o = torch.full_like(q, float("nan"))
    idx = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device="cuda")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    bra.bra_forward_lce(s, q, k, v, w_d, b_d, o, idx, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    idx_gpu = idx.cpu().numpy()
    qr = oracle.region_pool(inp.q_f64, shape.heads, shape.S)
    kr = oracle.region_pool(inp.k_f64, shape.heads, shape.S)
    rep = compare_routes(idx_gpu, oracle.region_affinity(qr, kr))
    assert not rep.mismatches, f"{len(rep.mismatches)} routing rows differ"
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx_gpu, shape.heads, shape.S)
    ref = ref + oracle.local_context(inp.v_f64, w.astype(np.float64), b.astype(np.float64) if b is not None else None)
    got = o.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), "some output was not written"
    err = np.abs(got - ref)
    bound = TOL[shape.dtype] + np.abs(ref) * 2.0 ** -8
    worst = float((err / bound).max())
    record_margin(label, float(err.max()), TOL[shape.dtype], rep.ambiguous, rep.rows)
    assert worst <= 1.0, f"max abs error {err.max():.3e}, worst error/bound {worst:.3f}"
    return worst


FUSED = {
    "stage1_b4": (4, 56, 56, 64, 2, 7, 1),          # the stage-1 shape: one route
    "stage1_full": (64, 56, 56, 64, 2, 7, 1),       # full size, the benchmark's launch configuration
    "topk4_regions8": (2, 64, 64, 64, 2, 8, 4),     # 8 x 8 regions, four routes (no 64-key fast path)
    "two_head_pairs": (2, 56, 56, 128, 4, 7, 2),    # channels 0-63 and 64-127 in separate tiles
    "edge_regions": (3, 16, 16, 64, 2, 2, 2),       # 2 x 2 regions: halos reach past every map edge
}


@pytest.mark.parametrize("name", list(FUSED))
def test_forward_lce_fused(name):
    check_forward_lce(bi.BraShape(*FUSED[name], "bf16"), 500 + len(name), f"{name} [fused lce]")


def test_forward_lce_without_bias():
    check_forward_lce(bi.BraShape(2, 56, 56, 64, 2, 7, 1, "bf16"), 541, "no_bias [fused lce]", with_bias=False)


@pytest.mark.parametrize("dims", [(2, 28, 28, 128, 4, 7, 4, "bf16"), (1, 16, 16, 64, 2, 4, 3, "f32")],
                         ids=["stage2_shape", "f32"])
def test_forward_lce_other_shapes(dims):
    """Shapes outside the fused epilogue: attention, then the filter."""
    shape = bi.BraShape(*dims)
    check_forward_lce(shape, 560 + shape.C, f"{shape.H}x{shape.W} C{shape.C} {shape.dtype} [lce after attention]")


def test_forward_lce_matches_attention_then_filter():
    """The fused result equals attention then bra_lce up to the one rounding
    the fused form saves (half a bf16 ulp of the attention result)."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(2, 56, 56, 64, 2, 7, 1, "bf16")
    inp = bi.make_inputs(shape, 77)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(2, 56, 56, 64, 2, 7, 1, "bf16")
    w, b = lce_params(64, 78)
    w_d, b_d = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    idx = torch.empty((2, 2, 49, 1), dtype=torch.int32, device="cuda")
    o1 = torch.empty_like(q)
    bra.bra_forward_lce(s, q, k, v, w_d, b_d, o1, idx, ws)
    o2 = torch.empty_like(q)
    bra.bra_forward(s, q, k, v, o2, idx, ws)
    bra.bra_lce(s, v, w_d, b_d, o2)
    torch.cuda.synchronize()
    a, c = o1.float(), o2.float()
    # two roundings against one: within one bf16 ulp of the result plus the attention's rounding
    assert ((a - c).abs() <= a.abs() * 2.0 ** -7 + 2.0 ** -7).all()
