"""bra_lce (local context enhancement: o += bias + 5x5 depthwise filter of v)
against the float64 oracle, through the C ABI.

Tolerance.  fp32: the 25 fp32 FMAs per output on O(1) values keep the error
near 1e-6; the test allows 1e-4 (the path's fp32 bound).  bf16: o is read as
bf16, the term is added in fp32 and the sum rounded once to bf16, so the
error is at most half a bf16 ulp of the result (|x| * 2^-9) plus the fp32
accumulation error; the test allows |x| * 2^-8 + 1e-3.
"""
import numpy as np
import pytest

import bra_inputs as bi
import oracle

pytestmark = pytest.mark.gpu


def run_case(B, H, W, C, dtype, seed, with_bias=True):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((B, H, W, C)).astype(np.float32)
    o = rng.standard_normal((B, H, W, C)).astype(np.float32)
    w = (rng.standard_normal((C, 5, 5)) / 5.0).astype(np.float32)
    b = rng.standard_normal(C).astype(np.float32) if with_bias else None
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    v_d = torch.from_numpy(v).to(tdt).cuda()
    o_d = torch.from_numpy(o).to(tdt).cuda()
    # the values the GPU reads, widened to float64
    v64 = v_d.double().cpu().numpy()
    o64 = o_d.double().cpu().numpy()
    w_d = torch.from_numpy(w).cuda()
    b_d = torch.from_numpy(b).cuda() if b is not None else None
    # heads/S/topk are only checked; any valid values do
    s = bra.shape_for(B, H, W, C, C // 32, 1, 1, dtype)
    bra.bra_lce(s, v_d, w_d, b_d, o_d)
    torch.cuda.synchronize()
    got = o_d.double().cpu().numpy()
    ref = o64 + oracle.local_context(v64, w.astype(np.float64), b.astype(np.float64) if b is not None else None)
    err = np.abs(got - ref)
    if dtype == "f32":
        assert err.max() <= 1e-4, err.max()
    else:
        bound = np.abs(ref) * 2.0 ** -8 + 1e-3
        assert (err <= bound).all(), f"max err {err.max():.3e}, worst ratio {(err / bound).max():.3f}"
    return err.max()


def test_lce_tiny_f32():
    run_case(1, 16, 16, 32, "f32", 1)


def test_lce_stage1_shape_bf16():
    run_case(8, 56, 56, 64, "bf16", 2)


@pytest.mark.parametrize("B,H,W,C,dtype", [
    (3, 13, 11, 32, "bf16"),   # ragged rows and columns, a half channel group
    (2, 7, 7, 512, "bf16"),    # many channel groups, map smaller than the filter reach
    (1, 5, 3, 96, "f32"),      # three fp32 channel groups, tiny map
    (2, 28, 28, 128, "bf16"),
])
def test_lce_shapes(B, H, W, C, dtype):
    run_case(B, H, W, C, dtype, B * 1000 + H * 10 + C)


def test_lce_without_bias():
    run_case(2, 14, 14, 64, "bf16", 7, with_bias=False)


def test_lce_empty_batch_is_a_no_op():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    s = bra.shape_for(0, 8, 8, 64, 2, 1, 1, "bf16")
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64 * 25, device="cuda")
    bra.bra_lce(s, t, w, None, t)
    torch.cuda.synchronize()
