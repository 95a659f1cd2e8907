"""Pins of the oracle's local context enhancement term (blog "BiFormer Reshapes
Visual Attention with Bi-Level Routing", Part 2 section 2.2, step 4 third
bullet and the "+ dwconv(value)" of pseudocode step 7): a 5x5 depthwise
filter of V, zero padding 2, cross-correlation orientation, plus a bias.

Each pin fixes the result by something other than the oracle's own loops: a
library routine (scipy's 2-D correlation), closed forms (identity, shifts,
constant input, bias only) and the linearity of the operation.  A second file
plants mistakes in the oracle's C source and checks that a pin fails."""
import numpy as np
import pytest
from scipy import signal

import oracle


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_matches_scipy_correlate2d_per_channel():
    v = rand((2, 9, 11, 5), 1)
    w = rand((5, 5, 5), 2)
    b = rand((5,), 3)
    out = oracle.local_context(v, w, b)
    for bb in range(2):
        for c in range(5):
            ref = signal.correlate2d(v[bb, :, :, c], w[c], mode="same", boundary="fill", fillvalue=0.0) + b[c]
            np.testing.assert_allclose(out[bb, :, :, c], ref, rtol=0, atol=1e-12)


def test_identity_kernel_returns_v():
    v = rand((1, 7, 6, 4), 4)
    w = np.zeros((4, 5, 5))
    w[:, 2, 2] = 1.0
    np.testing.assert_array_equal(oracle.local_context(v, w), v)


@pytest.mark.parametrize("dy,dx", [(-2, 0), (0, 2), (1, -1), (-2, -2), (2, 1)])
def test_single_tap_is_a_shift_with_zero_fill(dy, dx):
    """w[c, 2 + dy, 2 + dx] = 1 reads v[y + dy, x + dx] (cross-correlation), zero outside."""
    v = rand((1, 8, 9, 3), 5)
    w = np.zeros((3, 5, 5))
    w[:, 2 + dy, 2 + dx] = 1.0
    ref = np.zeros_like(v)
    H, W = 8, 9
    for y in range(H):
        for x in range(W):
            yy, xx = y + dy, x + dx
            if 0 <= yy < H and 0 <= xx < W:
                ref[0, y, x] = v[0, yy, xx]
    np.testing.assert_array_equal(oracle.local_context(v, w), ref)


def test_constant_input_gives_kernel_sums():
    """V = 1: interior = sum of all 25 taps + bias; a corner sees only the
    3 x 3 block of taps that stays inside; an edge middle a 3 x 5 block."""
    C = 3
    v = np.ones((1, 9, 9, C))
    w = rand((C, 5, 5), 6)
    b = rand((C,), 7)
    out = oracle.local_context(v, w, b)
    np.testing.assert_allclose(out[0, 4, 4], w.sum(axis=(1, 2)) + b, atol=1e-12)
    np.testing.assert_allclose(out[0, 0, 0], w[:, 2:, 2:].sum(axis=(1, 2)) + b, atol=1e-12)
    np.testing.assert_allclose(out[0, 8, 8], w[:, :3, :3].sum(axis=(1, 2)) + b, atol=1e-12)
    np.testing.assert_allclose(out[0, 0, 4], w[:, 2:, :].sum(axis=(1, 2)) + b, atol=1e-12)


def test_bias_only():
    v = rand((2, 5, 5, 4), 8)
    b = rand((4,), 9)
    out = oracle.local_context(v, np.zeros((4, 5, 5)), b)
    np.testing.assert_array_equal(out, np.broadcast_to(b, v.shape))


def test_linear_in_v_and_in_weights():
    v1, v2 = rand((1, 6, 7, 3), 10), rand((1, 6, 7, 3), 11)
    w1, w2 = rand((3, 5, 5), 12), rand((3, 5, 5), 13)
    f = oracle.local_context
    np.testing.assert_allclose(f(2.0 * v1 - 3.0 * v2, w1), 2.0 * f(v1, w1) - 3.0 * f(v2, w1), atol=1e-11)
    np.testing.assert_allclose(f(v1, 0.5 * w1 + w2), 0.5 * f(v1, w1) + f(v1, w2), atol=1e-11)


def test_channels_do_not_mix():
    v = rand((1, 6, 6, 4), 14)
    w = rand((4, 5, 5), 15)
    base = oracle.local_context(v, w)
    v2 = v.copy()
    v2[..., 1] += 10.0
    out = oracle.local_context(v2, w)
    for c in (0, 2, 3):
        np.testing.assert_array_equal(out[..., c], base[..., c])
    assert np.abs(out[..., 1] - base[..., 1]).max() > 1.0


def test_bad_sizes_raise():
    with pytest.raises(Exception):
        oracle.local_context(np.zeros((1, 0, 4, 2)), np.zeros((2, 5, 5)))
