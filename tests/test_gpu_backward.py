"""bra_attend_backward (dQ, dK, dV for a fixed routing) against the float64
oracle's gradients, through the C ABI, for both kernels
(BRA_BACKWARD_KERNEL pins one).

Tolerances.  Both kernels read exactly the values the oracle is given (bf16
inputs widened).

* "simt" (CUDA cores, fp32 throughout): the only differences are fp32
  rounding (dot products of 32 terms, softmax sums over at most 256 keys,
  dK/dV sums in any order), allowed as |err| <= 2e-4 * (1 + |ref|).
* "mma" (tensor cores): P and dS enter the products as bf16, each rounded
  once with relative error at most u = 2^-8, so
    |err dV_jc| <= u * sum_t P_tj |G_tc|
    |err dK_jc| <= u / sqrt(d) * sum_t |dS_tj| |Q_tc|
    |err dQ_tc| <= u / sqrt(d) * sum_j |dS_tj| |K_jc|
  plus the fp32 term above.  With |dP_tj| <= |G_t| |V_j| (Cauchy-Schwarz)
  and |D_t| <= max_j |dP_tj|, |dS_tj| <= 2 P_tj |G_t| Vmax (Vmax the
  largest |V_j| of the map), so every bound is a positive combination the
  oracle itself evaluates on transformed inputs: dV's is the oracle's dV for
  grad |G|, dK's its dV for grad |G_t| |Q_t|, dQ's its token attention
  with |K| in place of V.  No arithmetic of the oracle changes.
"""
import numpy as np
import pytest

import bra_inputs as bi
import oracle
from gpu_helpers import device_inputs
from parity import record_margin

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8


def run(shape: bi.BraShape, seed: int, kernel: str, monkeypatch, idx=None):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    if kernel:
        monkeypatch.setenv("BRA_BACKWARD_KERNEL", kernel)
    else:
        monkeypatch.delenv("BRA_BACKWARD_KERNEL", raising=False)
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
    # NaN-filled outputs: every element the kernel owes must be written
    dq, dk, dv = (torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda") for _ in range(3))
    bra.bra_attend_backward(s, q, k, v, idx_d, go, dq, dk, dv, ws)
    status = bra.bra_device_status(s, ws)
    torch.cuda.synchronize()
    g64 = go.double().cpu().numpy()
    idx_h = idx_d.cpu().numpy()
    ref = oracle.attention_backward(inp.q_f64, inp.k_f64, inp.v_f64, idx_h, g64, shape.heads,
                                    shape.S) if status == bra.BRA_OK else None
    got = tuple(t.double().cpu().numpy() for t in (dq, dk, dv))
    return status, got, ref, (inp, idx_h, g64)


def mma_bounds(shape: bi.BraShape, inp, idx, g64):
    """Per-element error bounds of the tensor-core kernel (module docstring)."""
    B, H, W, C, heads = shape.B, shape.H, shape.W, shape.C, shape.heads
    d = C // heads
    per_head = lambda x: x.reshape(B, H, W, heads, d)
    vmax = float(np.sqrt((per_head(inp.v_f64) ** 2).sum(-1)).max())
    gnorm = np.sqrt((per_head(g64) ** 2).sum(-1, keepdims=True))  # |G_t| per head
    q_abs, k_abs = np.abs(inp.q_f64), np.abs(inp.k_f64)
    _, _, dv_bound = oracle.attention_backward(inp.q_f64, inp.k_f64, inp.v_f64, idx, np.abs(g64), heads, shape.S)
    gq = (gnorm * per_head(q_abs)).reshape(B, H, W, C)
    _, _, dk_sum = oracle.attention_backward(inp.q_f64, inp.k_f64, inp.v_f64, idx, gq, heads, shape.S)
    pk = oracle.token_attention(inp.q_f64, inp.k_f64, k_abs, idx, heads, shape.S)
    dq_sum = (gnorm * per_head(pk)).reshape(B, H, W, C)
    scale = 1.0 / np.sqrt(d)
    return (U_BF16 * scale * 2.0 * vmax * dq_sum, U_BF16 * scale * 2.0 * vmax * dk_sum, U_BF16 * dv_bound)


def check(shape, got, ref, kernel, label, extra=None):
    worst = 0.0
    for i, (g_name, a, b) in enumerate(zip("qkv", got, ref)):
        assert np.isfinite(a).all(), f"d{g_name}: elements not written"
        err = np.abs(a - b)
        bound = 2e-4 * (1 + np.abs(b))
        if extra is not None:
            bound = bound + extra[i]
        ratio = float((err / bound).max())
        worst = max(worst, ratio)
        # recorded so that error / tolerance reads as the worst per-element ratio
        record_margin(f"backward {label} [{kernel}] d{g_name}", float(err.max()),
                      float(err.max()) / max(ratio, 1e-30))
        assert ratio <= 1.0, f"d{g_name}: max err {err.max():.3e}, worst err/bound {ratio:.3f}"
    return worst


SHAPES = {
    "tiny": bi.BraShape(1, 16, 16, 32, 1, 4, 2, "f32"),
    "stage1_b4": bi.BraShape(4, 56, 56, 64, 2, 7, 1, "bf16"),
    "stage2_b4": bi.BraShape(4, 28, 28, 128, 4, 7, 4, "bf16"),
    "stage3_b4": bi.BraShape(4, 14, 14, 256, 8, 7, 16, "bf16"),
    "dense_topk": bi.BraShape(1, 16, 16, 64, 2, 4, 16, "bf16"),
    "ragged": bi.BraShape(2, 24, 24, 64, 2, 4, 3, "f32"),
}

# shapes the tensor-core kernel covers: regions of 16..64 tokens in steps of
# 16, topk * n <= 128
MMA_SHAPES = {
    "stage1_b4": bi.BraShape(4, 56, 56, 64, 2, 7, 1, "bf16"),         # n 64, one route
    "stage2_b4": bi.BraShape(4, 28, 28, 128, 4, 7, 4, "bf16"),        # n 16, four routes
    "n32_topk4": bi.BraShape(2, 32, 16, 64, 2, 4, 4, "bf16"),         # 8 x 4 regions: n 32, 128 keys
    "n48_topk2": bi.BraShape(2, 24, 32, 64, 2, 4, 2, "bf16"),         # 6 x 8 regions: n 48, 96 keys
    "n64_topk2_heads3": bi.BraShape(2, 32, 32, 96, 3, 4, 2, "bf16"),  # odd head count, 128 keys
    "n16_topk8": bi.BraShape(1, 32, 32, 64, 2, 8, 8, "bf16"),         # eight routes of 16 tokens
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_simt_gradients_match_oracle(name, monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    status, got, ref, _ = run(SHAPES[name], 7, "simt", monkeypatch)
    assert status == bra.BRA_OK
    check(SHAPES[name], got, ref, "simt", name)


@pytest.mark.parametrize("name", list(MMA_SHAPES))
def test_mma_gradients_match_oracle(name, monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    shape = MMA_SHAPES[name]
    status, got, ref, (inp, idx, g64) = run(shape, 7, "mma", monkeypatch)
    assert status == bra.BRA_OK
    check(shape, got, ref, "mma", name, mma_bounds(shape, inp, idx, g64))


def test_mma_full_stage1(monkeypatch):
    """The benchmark's launch configuration (stage 1, 64 images), every output."""
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.WORKLOADS["stage1"][0]
    status, got, ref, (inp, idx, g64) = run(shape, 13, "mma", monkeypatch)
    assert status == bra.BRA_OK
    check(shape, got, ref, "mma", "stage1 (full size)", mma_bounds(shape, inp, idx, g64))


def test_auto_picks_a_kernel_for_every_shape(monkeypatch):
    """Without a pin every shape runs (tensor cores where covered)."""
    import dynamic_sparse_attention_bra_b200 as bra
    for name in ("stage1_b4", "stage3_b4"):
        status, got, ref, (inp, idx, g64) = run(SHAPES[name], 5, "", monkeypatch)
        assert status == bra.BRA_OK
        extra = mma_bounds(SHAPES[name], inp, idx, g64) if name == "stage1_b4" else None
        check(SHAPES[name], got, ref, "auto", name, extra)


def test_mma_pin_rejects_uncovered_shape(monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    with pytest.raises(bra.BraError):
        run(SHAPES["stage3_b4"], 7, "mma", monkeypatch)


@pytest.mark.parametrize("kernel", ["simt", "mma"])
def test_repeated_routes_count_once(kernel, monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(1, 16, 16, 64, 2, 4, 3, "bf16")  # n 16, 48 keys
    rng = np.random.default_rng(3)
    idx = rng.integers(0, shape.R, size=(shape.B, shape.heads, shape.R, shape.topk)).astype(np.int32)
    idx[..., 1] = idx[..., 0]  # every row lists a region twice
    idx[0, 0, 5, 2] = idx[0, 0, 5, 0]  # and one row three times
    status, got, ref, (inp, idx_h, g64) = run(shape, 9, kernel, monkeypatch, idx)
    assert status == bra.BRA_OK
    extra = mma_bounds(shape, inp, idx_h, g64) if kernel == "mma" else None
    check(shape, got, ref, kernel, "repeated routes", extra)


@pytest.mark.parametrize("kernel", ["simt", "mma"])
def test_out_of_range_route_is_reported(kernel, monkeypatch):
    """The region is skipped (its dq is zero, it adds nothing to dk, dv) and
    the status says so; every other region's gradients are exact."""
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(1, 16, 16, 64, 2, 4, 2, "bf16")
    rng = np.random.default_rng(4)
    idx = np.stack([rng.permutation(shape.R)[:shape.topk] for _ in range(shape.B * shape.heads * shape.R)])
    idx = idx.reshape(shape.B, shape.heads, shape.R, shape.topk).astype(np.int32)
    idx[0, 1, 3, 1] = shape.R + 5
    status, got, _, (inp, idx_h, g64) = run(shape, 11, kernel, monkeypatch, idx)
    assert status == bra.BRA_ERR_BAD_ROUTE
    # The reference: the same routing with region 3 of head 1 contributing
    # nothing.  With its G set to zero, dP and D vanish there, so its dS, its
    # dq rows and its share of dk, dv are zero in the oracle too.
    g_masked = g64.copy()
    hs, ws, d = shape.H // shape.S, shape.W // shape.S, shape.C // shape.heads
    ri, rj = divmod(3, shape.S)
    g_masked[0, ri * hs:(ri + 1) * hs, rj * ws:(rj + 1) * ws, d:2 * d] = 0.0
    idx_ok = idx_h.copy()
    idx_ok[0, 1, 3, 1] = idx_ok[0, 1, 3, 0]
    ref = oracle.attention_backward(inp.q_f64, inp.k_f64, inp.v_f64, idx_ok, g_masked, shape.heads, shape.S)
    extra = mma_bounds(shape, inp, idx_ok, g_masked) if kernel == "mma" else None
    check(shape, got, ref, kernel, "out-of-range route", extra)
