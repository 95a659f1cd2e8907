"""bra_qkv_project and bra_forward_qkv (the Q, K, V linear layer with the
region means fused into its epilogue, then routing and attention) against
the float64 oracle, through the C ABI.

Tolerances.  q, k, v: exact bf16 products summed in fp32 (C <= 128 terms of
O(1)), the bias added in fp32 and the result rounded once to bf16; the error
is half a bf16 ulp of the result (|ref| * 2^-9) plus the fp32 sum's, and the
test allows |ref| * 2^-8 + 1e-4.  q_r, k_r: the kernel averages its own bf16
q, the oracle averages its float64 q rounded to bf16; a value whose two
roundings differ moves one mean by at most one ulp / n, so the test allows
2^-8 * mean|q| + 1e-5 per region and channel.  Routing follows the
near-tie rule of tests/parity.py on the oracle's affinities; O is compared
with the oracle's attention on the GPU's own routing (bf16 bound 2e-2).
"""
import numpy as np
import pytest

import bra_inputs as bi
import oracle
from parity import TOL, compare_routes, record_margin

pytestmark = pytest.mark.gpu


def to_bf16_f64(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 (round to nearest even, through float32) -> float64."""
    return bi.bf16_bits_to_f64(bi.f32_to_bf16_bits(x.astype(np.float32)))


def oracle_projection(inp: bi.ProjectionInputs, with_bias: bool):
    q, k, v = oracle.qkv_projection(inp.x_f64, inp.w_f64, inp.b_f64 if with_bias else None)
    return q, k, v


def run(shape: bi.BraShape, seed: int, with_bias: bool = True, full_path: bool = False):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    inp = bi.make_projection_inputs(shape, seed)
    sh = shape
    x = torch.from_numpy(inp.x_store).view(torch.bfloat16).cuda()
    w = torch.from_numpy(inp.w_store).view(torch.bfloat16).cuda()
    b = torch.from_numpy(inp.b_store).cuda() if with_bias else None
    s = bra.shape_for(sh.B, sh.H, sh.W, sh.C, sh.heads, sh.S, sh.topk, "bf16")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    q, k, v = (torch.full_like(x, float("nan")) for _ in range(3))
    out = {}
    if full_path:
        o = torch.full_like(x, float("nan"))
        idx = torch.full((sh.B, sh.heads, sh.R, sh.topk), -1, dtype=torch.int32, device="cuda")
        bra.bra_forward_qkv(s, x, w, b, q, k, v, o, idx, ws)
        out["o"] = o.double().cpu().numpy()
        out["idx"] = idx.cpu().numpy()
    else:
        qr = torch.full((sh.B, sh.heads, sh.R, sh.d), float("nan"), device="cuda")
        kr = torch.full_like(qr, float("nan"))
        bra.bra_qkv_project(s, x, w, b, q, k, v, qr, kr, ws)
        out["qr"], out["kr"] = qr.double().cpu().numpy(), kr.double().cpu().numpy()
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    torch.cuda.synchronize()
    out["q"], out["k"], out["v"] = (t.double().cpu().numpy() for t in (q, k, v))
    return inp, out


def check_projection(inp, out, with_bias=True):
    refs = oracle_projection(inp, with_bias)
    for name, ref in zip("qkv", refs):
        got = out[name]
        err = np.abs(got - ref)
        bound = np.abs(ref) * 2.0 ** -8 + 1e-4
        assert (err <= bound).all(), f"{name}: max err {err.max():.3e}, worst ratio {(err / bound).max():.3f}"
    return refs


def check_means(inp, out, refs):
    sh = inp.shape
    for name, ref in (("qr", refs[0]), ("kr", refs[1])):
        rounded = to_bf16_f64(ref)
        want = oracle.region_pool(rounded, sh.heads, sh.S)
        scale = oracle.region_pool(np.abs(rounded), sh.heads, sh.S)
        err = np.abs(out[name] - want)
        bound = scale * 2.0 ** -8 + 1e-5
        assert (err <= bound).all(), f"{name}: max err {err.max():.3e}, worst ratio {(err / bound).max():.3f}"


SHAPES = {
    # B, H, W, C, heads, S, topk
    "full_width_bands": (2, 16, 16, 64, 2, 4, 2),
    "stage1_b2": (2, 56, 56, 64, 2, 7, 1),       # 16 x 8 boxes, last box of a band half outside
    "stage2_b2": (2, 28, 28, 128, 4, 7, 4),      # two channel blocks, 112-token boxes
    "detection": (1, 128, 128, 64, 2, 16, 4),
    "ragged_columns": (2, 40, 40, 64, 2, 5, 2),
    "one_token_regions": (3, 8, 8, 64, 2, 8, 3),
    "wide_regions": (1, 16, 48, 64, 2, 4, 3),    # 4 x 12 regions, 96-token boxes
    "last_band_outside": (1, 14, 14, 64, 2, 7, 5),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_projection_and_means(name):
    shape = bi.BraShape(*SHAPES[name], "bf16")
    inp, out = run(shape, 11 + len(name))
    refs = check_projection(inp, out)
    check_means(inp, out, refs)


def test_projection_without_bias():
    shape = bi.BraShape(2, 56, 56, 64, 2, 7, 1, "bf16")
    inp, out = run(shape, 5, with_bias=False)
    refs = check_projection(inp, out, with_bias=False)
    check_means(inp, out, refs)


@pytest.mark.parametrize("name", ["stage1_b2", "stage2_b2", "full_width_bands", "ragged_columns"])
def test_forward_from_feature_map(name):
    shape = bi.BraShape(*SHAPES[name], "bf16")
    inp, out = run(shape, 23 + len(name), full_path=True)
    refs = check_projection(inp, out)
    q, k, v = (to_bf16_f64(r) for r in refs)
    sh = shape
    qr, kr = oracle.region_pool(q, sh.heads, sh.S), oracle.region_pool(k, sh.heads, sh.S)
    rep = compare_routes(out["idx"], oracle.region_affinity(qr, kr))
    assert not rep.mismatches, rep.mismatches[:5]
    o_ref = oracle.token_attention(q, k, v, out["idx"], sh.heads, sh.S)
    err = float(np.abs(out["o"] - o_ref).max())
    record_margin(f"forward_qkv {name}", err, TOL["bf16"], rep.ambiguous, rep.rows)
    assert err <= TOL["bf16"], err


def test_stage1_full_size_projection_and_routing():
    # The workload the benchmark times (64 images of 56 x 56 x 64): every
    # q, k, v and mean is checked, and every routing row.
    shape = bi.WORKLOADS["stage1"][0]
    inp, out = run(shape, 101)
    refs = check_projection(inp, out)
    check_means(inp, out, refs)


def test_empty_batch_is_a_no_op():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    s = bra.shape_for(0, 56, 56, 64, 2, 7, 1, "bf16")
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    bra.bra_qkv_project(s, t, t, None, t, t, t, f, f, ws)
    torch.cuda.synchronize()
