"""The seeded input module shared by the oracle and the GPU tests: its random
numbers against the published generator, its bf16 rounding against a
library conversion, and its Gaussian recipe against closed forms."""
import numpy as np
import pytest

import bra_inputs as bi

MASK = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


def splitmix64_scalar(z: int) -> int:
    """The splitmix64 output function on one 64-bit word, in Python integers."""
    z &= MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def test_generator_reproduces_the_published_sequence():
    """With key 0 the counter form is the sequential generator started at
    state 0, whose first outputs are the published reference values."""
    z = np.array([(i + 1) * GOLDEN & MASK for i in range(3)], dtype=np.uint64)
    bi._mix(z, np.empty_like(z))
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_vectorised_stream_matches_scalar_across_a_chunk_boundary():
    count = bi._CHUNK + 7
    got = bi.splitmix_u64(3, 2, count)
    key = int(bi._key(3, 2))
    for i in (0, 1, 2, bi._CHUNK - 1, bi._CHUNK, bi._CHUNK + 6):
        assert int(got[i]) == splitmix64_scalar(key + (i + 1) * GOLDEN), i


def test_streams_and_seeds_differ():
    a, b, c = bi.splitmix_u64(1, 0, 64), bi.splitmix_u64(1, 1, 64), bi.splitmix_u64(2, 0, 64)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    np.testing.assert_array_equal(a, bi.splitmix_u64(1, 0, 64))


def test_uniform_is_open_interval_and_normal_moments():
    u = bi.uniform01(5, 0, 1 << 16)
    assert (u > 0).all() and (u < 1).all()
    n = bi.normal(5, 1, 1 << 18)
    # mean within 5 sigma of 0, variance within 5 sigma of 1 (sd of the sample variance ~ sqrt(2/N))
    assert abs(n.mean()) < 5.0 / np.sqrt(n.size)
    assert abs(n.var() - 1.0) < 5.0 * np.sqrt(2.0 / n.size)


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 4096),
                        # exact ties: mantissa low 16 bits = 0x8000, both parities of the kept bit
                        (np.arange(64, dtype=np.uint32) << 16 | 0x3F808000).view(np.float32),
                        (np.arange(64, dtype=np.uint32) << 17 | 0x3F818000).view(np.float32)])
    ours = bi.f32_to_bf16_bits(x).view(np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(bi.bf16_bits_to_f64(ours), torch.from_numpy(ref.view(np.int16)).view(
        torch.bfloat16).to(torch.float64).numpy())


def test_region_recipe_second_moments():
    """X = mu[region] + 0.5 eps: a token's variance is 1.25, two tokens of
    one region share mu (covariance 1), tokens of different regions do not."""
    shape = bi.BraShape(8, 32, 32, 64, 2, 4, 1, "f32")  # 16 regions of 8 x 8 tokens
    x = bi.make_inputs(shape, 11).q_f64  # [B, H, W, C]
    assert abs(x.var() - 1.25) < 0.05
    reg = bi.region_map(shape.H, shape.W, shape.S)
    prod = x[:, :, :-1, :] * x[:, :, 1:, :]  # horizontal neighbours
    same = reg[:, :-1] == reg[:, 1:]
    # averages over 8 x 16 x 64 = 8192 independent region means: standard error about 0.02
    assert abs(prod[:, same, :].mean() - 1.0) < 0.1
    assert abs(prod[:, ~same, :].mean()) < 0.1
