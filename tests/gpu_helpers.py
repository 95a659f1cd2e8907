"""Runs the CUDA path on seeded inputs and brings results back as numpy."""
from __future__ import annotations

import numpy as np

import bra_inputs as bi


def to_device(x: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.cuda()


def device_inputs(inp: bi.BraInputs):
    return [to_device(a, inp.shape.dtype) for a in (inp.q_store, inp.k_store, inp.v_store)]


def run_forward(inp: bi.BraInputs, check_status: bool = True):
    """bra_forward through the C ABI; returns (O as float64, I^r int32)."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    sh = inp.shape
    q, k, v = device_inputs(inp)
    shape = bra.shape_for(sh.B, sh.H, sh.W, sh.C, sh.heads, sh.S, sh.topk, sh.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    idx = torch.empty((sh.B, sh.heads, sh.R, sh.topk), dtype=torch.int32, device="cuda")
    bra.bra_forward(shape, q, k, v, o, idx, ws)
    if check_status:
        st = bra.bra_device_status(shape, ws)
        assert st == bra.BRA_OK, bra.bra_status_string(st)
    torch.cuda.synchronize()
    return o.float().cpu().numpy().astype(np.float64), idx.cpu().numpy()
