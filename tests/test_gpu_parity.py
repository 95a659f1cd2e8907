"""CUDA path vs the float64 oracle on the same seeded inputs, through the C ABI.

Routing is compared under the rule in ``parity.py`` (bit-exact wherever the
k-th/(k+1)-th affinity gap exceeds 1e-4 relative); O is compared with the
oracle's token attention on the GPU's routing, max-abs within 1e-4 (fp32)
or 2e-2 (bf16).  The five workload shapes run at full size, in the same
launch configuration the benchmark times; the extra shapes cover ragged
tiles, non-square regions, dense routing, a single region and the limits.
"""
import numpy as np
import pytest

import bra_inputs as bi
import oracle
from gpu_helpers import device_inputs, run_forward
from parity import TOL, compare_routes, record_margin

pytestmark = pytest.mark.gpu


def check_case(shape: bi.BraShape, seed: int, max_ambiguous_frac: float = 0.01, label: str | None = None):
    inp = bi.make_inputs(shape, seed)
    o_gpu, idx_gpu = run_forward(inp)
    qr = oracle.region_pool(inp.q_f64, shape.heads, shape.S)
    kr = oracle.region_pool(inp.k_f64, shape.heads, shape.S)
    a = oracle.region_affinity(qr, kr)
    rep = compare_routes(idx_gpu, a)
    assert not rep.mismatches, f"{len(rep.mismatches)} routing rows differ, first {rep.mismatches[:3]}"
    assert rep.ambiguous <= max(1, max_ambiguous_frac * rep.rows), rep.ambiguous
    o_ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx_gpu, shape.heads, shape.S)
    err = float(np.abs(o_gpu - o_ref).max())
    record_margin(label or str(shape), err, TOL[shape.dtype], rep.ambiguous, rep.rows)
    assert err <= TOL[shape.dtype], f"max abs error {err:.3e} > {TOL[shape.dtype]}"
    # the oracle's own routing gives the same O wherever the sets agree
    return err, rep


@pytest.mark.parametrize("name", list(bi.WORKLOADS))
def test_workloads_full_size(name):
    shape, seed = bi.WORKLOADS[name]
    check_case(shape, seed, label=f"{name} (full size)")


@pytest.fixture
def pinned_kernel(request, monkeypatch):
    """Pins the attention kernel through BRA_ATTEND_KERNEL for one test."""
    monkeypatch.setenv("BRA_ATTEND_KERNEL", request.param)
    return request.param


# Every attention kernel on every shape it covers (the default run above uses
# the first kernel that covers each shape).
KERNEL_CASES = [(k, w) for k in ("slice", "warp", "flash", "stack", "tiled", "simt")
                for w in ("stage1", "stage2", "stage3", "highres")]


@pytest.mark.parametrize("pinned_kernel,name", KERNEL_CASES, indirect=["pinned_kernel"],
                         ids=[f"{k}-{w}" for k, w in KERNEL_CASES])
def test_each_kernel_on_workloads(pinned_kernel, name):
    import dynamic_sparse_attention_bra_b200 as bra
    shape, seed = bi.WORKLOADS[name]
    try:
        check_case(shape, seed, label=f"{name} [{pinned_kernel}]")
    except bra.BraError as e:
        if e.status != bra.BRA_ERR_UNSUPPORTED:
            raise
        assert pinned_kernel != "simt"
        assert (pinned_kernel, name) not in (("warp", "stage2"), ("slice", "stage3"), ("flash", "highres"))
        pytest.skip(f"{pinned_kernel} does not cover {name}")


EXTRA = {
    # name: (B, H, W, C, heads, S, topk, dtype)
    "ragged_bf16": (2, 24, 24, 64, 2, 4, 3, "bf16"),        # n = 36: partial tiles
    "ragged_f32": (2, 24, 24, 64, 2, 4, 3, "f32"),
    "nonsquare_regions": (1, 18, 12, 32, 1, 6, 5, "bf16"),  # 3x2 tokens per region
    "wide_map": (1, 16, 48, 64, 2, 4, 2, "bf16"),           # 4x12 tokens per region
    "wide_map_batch": (24, 16, 48, 64, 2, 4, 2, "bf16"),    # the same, several tiles per CTA
    "dense_topk": (1, 16, 16, 64, 2, 4, 16, "bf16"),        # k = S^2: full attention
    "single_region": (2, 16, 20, 64, 2, 1, 1, "bf16"),      # n = 320: several query tiles
    "single_token_regions": (2, 8, 8, 64, 2, 8, 4, "bf16"), # n = 1
    "max_regions": (1, 32, 32, 32, 1, 16, 8, "bf16"),       # R = 256
    "many_heads": (1, 14, 14, 512, 16, 7, 16, "bf16"),
    "long_route_f32": (1, 32, 32, 32, 1, 4, 12, "f32"),     # 768 keys per query
    # S / k ablation of the BiFormer pages (per-image geometry of each stage, batch 8):
    # S = 7 with k = [1, 2, 8, 32] and S = [8, 4, 2, 1] with k = [2, 2, 2, 1]
    "ablation_k2_stage2": (8, 28, 28, 128, 4, 7, 2, "bf16"),   # 32 keys per query
    "ablation_k8_stage3": (8, 14, 14, 256, 8, 7, 8, "bf16"),   # 32 keys per query
    "ablation_k32_stage4": (8, 7, 7, 512, 16, 7, 32, "bf16"),  # one-token regions
    "stage4_full": (8, 7, 7, 512, 16, 7, 49, "bf16"),          # k = S^2: full attention
    "ablation_s8_stage1": (8, 56, 56, 64, 2, 8, 2, "bf16"),    # 49-token regions, 98 keys
    "ablation_s4_stage2": (8, 28, 28, 128, 4, 4, 2, "bf16"),
    "ablation_s2_stage3": (8, 14, 14, 256, 8, 2, 2, "bf16"),
    "ablation_s1_stage4": (8, 7, 7, 512, 16, 1, 1, "bf16"),    # one region: dense
    "three_heads": (4, 28, 28, 96, 3, 7, 4, "bf16"),           # 12 vectors per token: region-form pooling
}


@pytest.mark.parametrize("name", list(EXTRA))
def test_extra_shapes(name):
    B, H, W, C, heads, S, topk, dtype = EXTRA[name]
    check_case(bi.BraShape(B, H, W, C, heads, S, topk, dtype), 100 + len(name), label=name)


def test_repeatable_bitwise():
    shape, seed = bi.WORKLOADS["stage2"]
    inp = bi.make_inputs(shape, seed)
    o1, i1 = run_forward(inp)
    o2, i2 = run_forward(inp)
    assert (i1 == i2).all() and (o1 == o2).all()


def test_route_then_attend_equals_forward():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape, seed = bi.WORKLOADS["stage3"]
    inp = bi.make_inputs(shape, seed)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    bra.bra_route(s, q, k, idx, ws)
    bra.bra_attend(s, q, k, v, idx, o, ws)
    o2, idx2 = bra.forward(q, k, v, shape.heads, shape.S, shape.topk)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(o.view(torch.int16), o2.view(torch.int16))


def test_attend_with_given_routing():
    """bra_attend takes any routing, e.g. the oracle's own."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(2, 16, 16, 64, 2, 4, 3, "bf16")
    inp = bi.make_inputs(shape, 9)
    _, idx_or = oracle.bra_forward(inp.q_f64, inp.k_f64, inp.v_f64, shape.heads, shape.S, shape.topk)
    idx_or = np.ascontiguousarray(idx_or[..., ::-1])  # any order is a valid routing
    q, k, v = device_inputs(inp)
    s = bra.shape_for(*[getattr(shape, f) for f in "B H W C heads S topk".split()], shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    bra.bra_attend(s, q, k, v, torch.from_numpy(idx_or).cuda(), o, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    o_ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx_or, shape.heads, shape.S)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_repeated_routes_attend_the_union(dtype):
    """A caller-given routing that repeats a region in a row: every routed
    region's tokens count once (both the tensor-core and the fp32 kernel)."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(1, 16, 16, 32, 1, 4, 3, dtype)
    inp = bi.make_inputs(shape, 12)
    rng = np.random.default_rng(0)
    idx = rng.integers(0, 16, size=(1, 1, 16, 3)).astype(np.int32)
    idx[0, 0, :4] = [[2, 2, 2], [5, 1, 5], [0, 0, 7], [9, 3, 3]]
    q, k, v = device_inputs(inp)
    s = bra.shape_for(1, 16, 16, 32, 1, 4, 3, dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    bra.bra_attend(s, q, k, v, torch.from_numpy(idx).cuda(), o, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx, 1, 4)
    err = float(np.abs(o.float().cpu().numpy() - ref).max())
    record_margin(f"repeated_routes_{dtype}", err, TOL[dtype], 0, 16)
    assert err <= TOL[dtype]


@pytest.mark.parametrize("bad_value", [-1, 16, 1 << 30])
def test_bad_route_is_reported_not_read(bad_value):
    """An out-of-range routing index is caught by the kernel's own check: the
    region is skipped and the status block says BRA_ERR_BAD_ROUTE."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape = bi.BraShape(1, 16, 16, 64, 2, 4, 2, "bf16")
    inp = bi.make_inputs(shape, 3)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(1, 16, 16, 64, 2, 4, 2, "bf16")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    idx = torch.zeros((1, 2, 16, 2), dtype=torch.int32, device="cuda")
    idx[0, 1, 5, 1] = bad_value
    o = torch.zeros_like(q)
    bra.bra_attend(s, q, k, v, idx, o, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_ERR_BAD_ROUTE
    assert bra.bra_device_status(s, ws) == bra.BRA_OK  # cleared by the read


def test_empty_batch_is_a_noop():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    s = bra.shape_for(0, 56, 56, 64, 2, 7, 1, "bf16")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    buf = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(4, dtype=torch.int32, device="cuda")
    bra.bra_forward(s, buf, buf, buf, buf, idx, ws)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK


# The persistent kernel with each number of softmax warp groups (1, 2, 4) on
# the shapes it covers: 64-key windows with one and with four query regions
# per half, and 96-key windows (the masked softmax path).
GROUP_CASES = [(gr, w) for gr in (1, 2, 4) for w in ("stage1", "stage2", "wide_map_batch")]


@pytest.mark.parametrize("groups,name", GROUP_CASES, ids=[f"groups{g}-{w}" for g, w in GROUP_CASES])
def test_stack_kernel_groups(groups, name, monkeypatch):
    monkeypatch.setenv("BRA_ATTEND_KERNEL", "stack")
    monkeypatch.setenv("BRA_STACK_GROUPS", str(groups))
    if name in bi.WORKLOADS:
        shape, seed = bi.WORKLOADS[name]
    else:
        B, H, W, C, heads, S, topk, dtype = EXTRA[name]
        shape, seed = bi.BraShape(B, H, W, C, heads, S, topk, dtype), 11
    check_case(shape, seed, label=f"{name} [stack, {groups} groups]")


def test_workspace_reused_across_calls():
    """One workspace serves any number of ordered calls: each call on a reused
    workspace gives bit-identical results to the same call on a fresh one."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    from gpu_helpers import device_inputs
    shape, _ = bi.WORKLOADS["stage2"]
    sh = bi.BraShape(8, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    s = bra.shape_for(sh.B, sh.H, sh.W, sh.C, sh.heads, sh.S, sh.topk, sh.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    for seed in (21, 22, 23):
        inp = bi.make_inputs(sh, seed)
        q, k, v = device_inputs(inp)
        o = torch.empty_like(q)
        idx = torch.empty((sh.B, sh.heads, sh.R, sh.topk), dtype=torch.int32, device="cuda")
        bra.bra_forward(s, q, k, v, o, idx, ws)
        assert bra.bra_device_status(s, ws) == bra.BRA_OK
        torch.cuda.synchronize()
        # the same call on a fresh workspace gives bit-identical results
        ws2 = torch.zeros_like(ws)
        o2 = torch.empty_like(q)
        idx2 = torch.empty_like(idx)
        bra.bra_forward(s, q, k, v, o2, idx2, ws2)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx2)
        assert torch.equal(o.view(torch.int16), o2.view(torch.int16))


# The resident-slice warp kernel on the shapes it covers: several routes of
# 16 or 32 tokens, 64 and 128 keys per query region, one image, many slices.
WARP_CASES = {
    "stage2_batch8": (8, 28, 28, 128, 4, 7, 4),
    "stage2_one_image": (1, 28, 28, 128, 4, 7, 4),      # 4 slices: most CTAs idle
    "topk8_128_keys": (4, 28, 28, 128, 4, 7, 8),        # two query regions per half
    "regions_of_32": (4, 32, 16, 64, 2, 4, 2),          # 8 x 4 regions, R = 16
    "odd_heads": (3, 28, 28, 96, 3, 7, 4),
    "many_slices": (150, 28, 28, 32, 1, 7, 4),          # 150 slices: two for some CTAs
}


@pytest.mark.parametrize("kernel", ["warp"])
@pytest.mark.parametrize("name", list(WARP_CASES))
def test_warp_kernel(name, kernel, monkeypatch):
    monkeypatch.setenv("BRA_ATTEND_KERNEL", kernel)
    B, H, W, C, heads, S, topk = WARP_CASES[name]
    check_case(bi.BraShape(B, H, W, C, heads, S, topk, "bf16"), 200 + len(name), label=f"{name} [{kernel}]")


def attend_given_routes(shape, seed, idx):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    inp = bi.make_inputs(shape, seed)
    q, k, v = device_inputs(inp)
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    o = torch.zeros_like(q)
    bra.bra_attend(s, q, k, v, torch.from_numpy(idx).cuda(), o, ws)
    status = bra.bra_device_status(s, ws)
    return inp, o.float().cpu().numpy(), status


@pytest.mark.parametrize("kernel", ["warp"])
def test_warp_repeated_routes_attend_the_union(kernel, monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    monkeypatch.setenv("BRA_ATTEND_KERNEL", kernel)
    shape = bi.BraShape(2, 28, 28, 64, 2, 7, 4, "bf16")
    rng = np.random.default_rng(5)
    idx = rng.integers(0, shape.R, size=(shape.B, shape.heads, shape.R, shape.topk)).astype(np.int32)
    idx[0, 0, :3] = [[3, 3, 3, 3], [7, 1, 7, 2], [0, 0, 48, 48]]
    inp, o, status = attend_given_routes(shape, 13, idx)
    assert status == bra.BRA_OK
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx, shape.heads, shape.S)
    err = float(np.abs(o - ref).max())
    record_margin(f"repeated_routes [{kernel}]", err, TOL["bf16"])
    assert err <= TOL["bf16"]


@pytest.mark.parametrize("kernel", ["warp"])
@pytest.mark.parametrize("bad_value", [-1, 49, 1 << 30])
def test_warp_bad_route_is_reported_not_read(bad_value, kernel, monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    monkeypatch.setenv("BRA_ATTEND_KERNEL", kernel)
    shape = bi.BraShape(1, 28, 28, 64, 2, 7, 4, "bf16")
    idx = np.tile(np.arange(4, dtype=np.int32), (1, 2, 49, 1))
    idx[0, 1, 20, 2] = bad_value
    inp, o, status = attend_given_routes(shape, 4, idx)
    assert status == bra.BRA_ERR_BAD_ROUTE
    # every other region is still attended correctly
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, np.where(idx < 0, 0, np.minimum(idx, 48)),
                                 shape.heads, shape.S)
    reg = bi.region_map(shape.H, shape.W, shape.S)
    keep = np.ones(o.shape, dtype=bool)
    keep[0][reg == 20, 32:64] = False
    assert np.abs(o - ref)[keep].max() <= TOL["bf16"]


# The dense-slice kernel on the maps it covers (at most 256 tokens per
# (batch, head)): one and two 128-query units per slice, regions of one to
# sixteen tokens, routes up to S^2, bad and repeated routes.
SLICE_CASES = {
    "stage3_batch8": (8, 14, 14, 256, 8, 7, 16),
    "stage4_full": (8, 7, 7, 512, 16, 7, 49),           # one-token regions, k = S^2
    "map_16x12": (3, 16, 12, 64, 2, 4, 3),              # 192 tokens, 4 x 3 regions
    "map_12x10": (5, 12, 10, 96, 3, 2, 1),              # 120 tokens: one unit, 6 x 5 regions
    "one_region": (2, 8, 8, 64, 2, 1, 1),               # S = 1: dense attention
    "many_slices": (40, 14, 14, 256, 8, 7, 4),          # 320 slices
}


@pytest.mark.parametrize("name", list(SLICE_CASES))
def test_slice_kernel(name, monkeypatch):
    monkeypatch.setenv("BRA_ATTEND_KERNEL", "slice")
    B, H, W, C, heads, S, topk = SLICE_CASES[name]
    check_case(bi.BraShape(B, H, W, C, heads, S, topk, "bf16"), 300 + len(name), label=f"{name} [slice]")


def test_slice_repeated_and_bad_routes(monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    monkeypatch.setenv("BRA_ATTEND_KERNEL", "slice")
    shape = bi.BraShape(2, 14, 14, 64, 2, 7, 5, "bf16")
    rng = np.random.default_rng(8)
    idx = rng.integers(0, shape.R, size=(shape.B, shape.heads, shape.R, shape.topk)).astype(np.int32)
    idx[0, 0, :3] = [[3, 3, 3, 3, 3], [7, 1, 7, 2, 1], [0, 0, 48, 48, 9]]
    inp, o, status = attend_given_routes(shape, 17, idx)
    assert status == bra.BRA_OK
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx, shape.heads, shape.S)
    err = float(np.abs(o - ref).max())
    record_margin("repeated_routes [slice]", err, TOL["bf16"])
    assert err <= TOL["bf16"]
    bad = idx.copy()
    bad[1, 1, 30, 4] = 49
    inp, o, status = attend_given_routes(shape, 17, bad)
    assert status == bra.BRA_ERR_BAD_ROUTE
    reg = bi.region_map(shape.H, shape.W, shape.S)
    skipped = np.zeros(o.shape, dtype=bool)
    skipped[1][reg == 30, 32:64] = True
    assert (o[skipped] == 0).all()  # the region's outputs are left as they were
    assert np.abs(o - ref)[~skipped & (np.arange(shape.B) == 1)[:, None, None, None]].max() <= TOL["bf16"]


# The flash kernel on the shapes it covers (regions of a multiple of 128
# tokens): 256- and 128-token regions, two and eight key blocks per tile,
# one route, k = S^2, an odd number of tiles per CTA.
FLASH_CASES = {
    "highres_b1": (1, 128, 128, 64, 2, 8, 4),
    "regions_128": (2, 64, 32, 64, 2, 4, 3),          # 16 x 8 regions: one block per route
    "one_route": (2, 64, 64, 64, 2, 4, 1),
    "dense_k": (1, 32, 64, 64, 2, 2, 4),              # 16 x 32 regions, k = S^2
    "odd_tiles": (1, 64, 64, 96, 3, 4, 2),            # 3 heads: tiles not a multiple of the grid
    "regions_384": (1, 48, 32, 64, 2, 2, 2),          # 24 x 16 regions: three query tiles per region
}


@pytest.mark.parametrize("name", list(FLASH_CASES))
def test_flash_kernel(name, monkeypatch):
    monkeypatch.setenv("BRA_ATTEND_KERNEL", "flash")
    B, H, W, C, heads, S, topk = FLASH_CASES[name]
    check_case(bi.BraShape(B, H, W, C, heads, S, topk, "bf16"), 400 + len(name), label=f"{name} [flash]")


# 256-token regions (two query tiles and two key blocks per region) and
# 128-token regions (one of each)
@pytest.mark.parametrize("dims", [(1, 64, 64, 64, 2, 4, 3), (1, 64, 32, 64, 2, 4, 3)],
                         ids=["regions_256", "regions_128"])
def test_flash_repeated_and_bad_routes(dims, monkeypatch):
    import dynamic_sparse_attention_bra_b200 as bra
    monkeypatch.setenv("BRA_ATTEND_KERNEL", "flash")
    shape = bi.BraShape(*dims, "bf16")
    rng = np.random.default_rng(9)
    idx = rng.integers(0, shape.R, size=(shape.B, shape.heads, shape.R, shape.topk)).astype(np.int32)
    idx[0, 0, :3] = [[3, 3, 3], [7, 1, 7], [0, 15, 15]]
    inp, o, status = attend_given_routes(shape, 19, idx)
    assert status == bra.BRA_OK
    ref = oracle.token_attention(inp.q_f64, inp.k_f64, inp.v_f64, idx, shape.heads, shape.S)
    err = float(np.abs(o - ref).max())
    record_margin(f"repeated_routes [flash, {shape.H}x{shape.W}]", err, TOL["bf16"])
    assert err <= TOL["bf16"]
    bad = idx.copy()
    bad[0, 1, 5, 2] = -3
    inp, o, status = attend_given_routes(shape, 19, bad)
    assert status == bra.BRA_ERR_BAD_ROUTE
    reg = bi.region_map(shape.H, shape.W, shape.S)
    skipped = np.zeros(o.shape, dtype=bool)
    skipped[0][reg == 5, 32:64] = True
    assert (o[skipped] == 0).all()
    assert np.abs(o - ref)[~skipped].max() <= TOL["bf16"]
