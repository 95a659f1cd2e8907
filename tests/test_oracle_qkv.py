"""Pins of the oracle's linear projection (blog "BiFormer Reshapes Visual
Attention with Bi-Level Routing", Part 2 section 2.2, step 2 and pseudocode
step 2): Q, K, V are the three channel chunks, in that order, of one linear
layer x W^T + b applied to every token.

Each pin fixes the result by something other than the oracle's own loops:
closed forms (block identities, a channel permutation, bias only), a library
routine (numpy's matmul), the locality of a per-token map, and the identity
that the region mean of a linear map is the linear map of the region mean,
which ties the projection to the already pinned pooling step.  A second file
plants mistakes in the oracle's C source and checks that a pin fails."""
import numpy as np
import pytest

import oracle


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_block_identity_weights_give_scaled_copies():
    C = 6
    x = rand((2, 4, 5, C), 1)
    eye = np.eye(C)
    w = np.concatenate([eye, 2.0 * eye, -3.0 * eye], axis=0)  # [3C, C]
    q, k, v = oracle.qkv_projection(x, w)
    np.testing.assert_array_equal(q, x)
    np.testing.assert_array_equal(k, 2.0 * x)
    np.testing.assert_array_equal(v, -3.0 * x)


def test_bias_only_fills_each_chunk_with_its_bias():
    C = 5
    x = rand((1, 3, 3, C), 2)
    b = rand((3 * C,), 3)
    q, k, v = oracle.qkv_projection(x, np.zeros((3 * C, C)), b)
    np.testing.assert_array_equal(q, np.broadcast_to(b[:C], q.shape))
    np.testing.assert_array_equal(k, np.broadcast_to(b[C:2 * C], k.shape))
    np.testing.assert_array_equal(v, np.broadcast_to(b[2 * C:], v.shape))


def test_permutation_rows_select_input_channels():
    # Row o of the weight picks input channel pi(o): output channel o of each
    # chunk must equal x[..., pi(o)] (a transposed weight would give pi^-1).
    C = 7
    x = rand((1, 2, 3, C), 4)
    pis = [np.array([1, 2, 0, 4, 5, 6, 3]), np.array([6, 0, 1, 2, 3, 4, 5]),
           np.array([2, 0, 1, 6, 3, 4, 5])]
    w = np.zeros((3 * C, C))
    for j, pi in enumerate(pis):
        w[j * C + np.arange(C), pi] = 1.0
    outs = oracle.qkv_projection(x, w)
    for out, pi in zip(outs, pis):
        np.testing.assert_array_equal(out, x[..., pi])


@pytest.mark.parametrize("with_bias", [False, True])
def test_matches_numpy_matmul(with_bias):
    C = 16
    x = rand((2, 6, 4, C), 5)
    w = rand((3 * C, C), 6)
    b = rand((3 * C,), 7) if with_bias else None
    ref = x.reshape(-1, C) @ w.T + (b if with_bias else 0.0)
    got = np.concatenate(oracle.qkv_projection(x, w, b), axis=-1).reshape(-1, 3 * C)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_token_locality():
    # Changing one token changes that token's q, k, v and nothing else.
    C = 8
    x = rand((1, 4, 4, C), 8)
    w, b = rand((3 * C, C), 9), rand((3 * C,), 10)
    base = oracle.qkv_projection(x, w, b)
    x2 = x.copy()
    x2[0, 2, 1] += rand((C,), 11)
    moved = oracle.qkv_projection(x2, w, b)
    for a, m in zip(base, moved):
        diff = np.abs(a - m).max(axis=-1)[0]
        assert diff[2, 1] > 0
        diff[2, 1] = 0
        assert not diff.any()


def test_region_mean_of_projection_is_projection_of_region_mean():
    # mean_region(x W_q^T + b_q) = mean_region(x) W_q^T + b_q, tying the
    # projection to the pinned pooling step that routing reads.
    B, H, W, C, heads, S = 2, 8, 12, 8, 2, 4
    x = rand((B, H, W, C), 12)
    w, b = rand((3 * C, C), 13), rand((3 * C,), 14)
    q, k, _ = oracle.qkv_projection(x, w, b)
    xr = oracle.region_pool(x, 1, S)[:, 0]  # [B, R, C], one head holding every channel
    for j, out in enumerate((q, k)):
        ref = xr @ w[j * C:(j + 1) * C].T + b[j * C:(j + 1) * C]  # [B, R, C]
        got = oracle.region_pool(out, heads, S)  # [B, heads, R, d]
        got = np.transpose(got, (0, 2, 1, 3)).reshape(B, S * S, C)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
