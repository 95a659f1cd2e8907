"""Pins of the oracle's attention gradients (the backward of blog "BiFormer
Reshapes Visual Attention with Bi-Level Routing", Part 2 section 2.2 step 4,
for a fixed routing I^r).

They fix the result by computations independent of the backward loops:
central finite differences of the forward oracle (for L = sum O * G), torch
float64 autograd on dense attention when topk = S^2 (every region routed), and
autograd on a region-masked dense formulation, which also pins the reading
that a region listed twice in a routing row counts once."""
import numpy as np
import pytest
import torch

import oracle


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def routed(q, k, heads, S, topk):
    qr = oracle.region_pool(q, heads, S)
    kr = oracle.region_pool(k, heads, S)
    return oracle.topk_routing(oracle.region_affinity(qr, kr), topk)


@pytest.mark.parametrize("B,H,W,C,heads,S,topk", [(1, 4, 4, 4, 1, 2, 2), (2, 6, 4, 6, 2, 2, 3), (1, 4, 6, 4, 2, 2, 1)])
def test_gradients_match_finite_differences(B, H, W, C, heads, S, topk):
    q, k, v = rand((B, H, W, C), 1), rand((B, H, W, C), 2), rand((B, H, W, C), 3)
    g = rand((B, H, W, C), 4)
    idx = routed(q, k, heads, S, topk)
    dq, dk, dv = oracle.attention_backward(q, k, v, idx, g, heads, S)

    def loss(qq, kk, vv):
        return float((oracle.token_attention(qq, kk, vv, idx, heads, S) * g).sum())

    h = 1e-6
    rng = np.random.default_rng(5)
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            i = tuple(int(rng.integers(0, sz)) for sz in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[i] += h
            xm[i] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(num - grad[i]) < 1e-6 * (1 + abs(num)), (name, i, num, grad[i])


def dense_reference(q, k, v, g, heads, mask=None):
    """Autograd (float64) of per-head dense softmax(Q K^T / sqrt(d)) V, optionally
    with a [B, heads, HW, HW] boolean mask of allowed keys."""
    B, H, W, C = q.shape
    d = C // heads
    tq, tk, tv = (torch.tensor(x.reshape(B, H * W, heads, d).transpose(0, 2, 1, 3), requires_grad=True)
                  for x in (q, k, v))
    s = tq @ tk.transpose(-1, -2) / np.sqrt(d)
    if mask is not None:
        s = s.masked_fill(~torch.tensor(mask), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    tg = torch.tensor(g.reshape(B, H * W, heads, d).transpose(0, 2, 1, 3))
    (o * tg).sum().backward()
    back = lambda t: t.grad.numpy().transpose(0, 2, 1, 3).reshape(B, H, W, C)
    return back(tq), back(tk), back(tv)


def test_full_routing_is_dense_attention_gradient():
    B, H, W, C, heads, S = 1, 4, 4, 8, 2, 2
    q, k, v, g = rand((B, H, W, C), 6), rand((B, H, W, C), 7), rand((B, H, W, C), 8), rand((B, H, W, C), 9)
    idx = routed(q, k, heads, S, S * S)
    got = oracle.attention_backward(q, k, v, idx, g, heads, S)
    ref = dense_reference(q, k, v, g, heads)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, atol=1e-12)


def region_of(H, W, S):
    hs, ws = H // S, W // S
    return np.array([(y // hs) * S + (x // ws) for y in range(H) for x in range(W)])


def test_repeated_routes_count_once_like_a_masked_dense_attention():
    B, H, W, C, heads, S = 1, 4, 4, 4, 1, 2
    q, k, v, g = rand((B, H, W, C), 10), rand((B, H, W, C), 11), rand((B, H, W, C), 12), rand((B, H, W, C), 13)
    idx = np.array([[[[1, 1, 3], [0, 2, 0], [2, 2, 2], [3, 0, 1]]]], dtype=np.int32)  # [B, heads, R, topk]
    got = oracle.attention_backward(q, k, v, idx, g, heads, S)
    reg = region_of(H, W, S)
    mask = np.zeros((B, heads, H * W, H * W), dtype=bool)
    for t in range(H * W):
        for m in idx[0, 0, reg[t]]:
            mask[0, 0, t, reg == m] = True
    ref = dense_reference(q, k, v, g, heads, mask)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, atol=1e-12)


def test_zero_incoming_gradient_gives_zero_gradients():
    q, k, v = rand((1, 4, 4, 4), 14), rand((1, 4, 4, 4), 15), rand((1, 4, 4, 4), 16)
    idx = routed(q, k, 1, 2, 2)
    for x in oracle.attention_backward(q, k, v, idx, np.zeros_like(q), 1, 2):
        assert not x.any()
