"""The pins have teeth: each plausible slip, planted in a copy of the oracle's
C source and compiled on the CPU, must make at least one pin test fail."""
import os
import subprocess

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "bra_oracle.c")

# (name, original text, mutated text)
MUTATIONS = [
    ("no_softmax_scale", "double scale = 1.0 / sqrt((double)d);", "double scale = 1.0;"),
    ("pool_sum_not_mean", "= sum / (double)n;", "= sum;"),
    ("affinity_transposed",
     "a[((size_t)bh * R + r) * R + s] = dot;", "a[((size_t)bh * R + s) * R + r] = dot;"),
    ("tie_to_higher_index",
     "return (a->index > b->index) - (a->index < b->index);",
     "return (a->index < b->index) - (a->index > b->index);"),
    ("topk_smallest_first", "if (a->value > b->value) return -1;", "if (a->value < b->value) return -1;"),
    ("region_column_major", "int ri = r / S, rj = r % S;", "int ri = r % S, rj = r / S;"),
    ("token_column_major", "*y = ri * hs + t / ws;", "*y = ri * hs + t % hs;"),
    ("softmax_weights_perturbed", "s[j] = exp(s[j] - mx);", "s[j] = exp(s[j] - mx + 1e-3 * j);"),
    ("values_from_keys", "num += s[j] * v[key_off[j] + c];", "num += s[j] * k[key_off[j] + c];"),
    ("first_route_only", "int rr = route[m];", "int rr = route[0];"),
    ("repeats_counted_twice", "                    if (listed_before) continue;\n", ""),
]


def build_variant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation {name}: anchor text not found exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", str(lib), str(path), "-lm"])
    return str(lib)


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, name, old, new):
    import test_oracle_pins as pins
    lib = build_variant(tmp_path, name, old, new)
    checks = [
        pins.test_region_pool_is_block_mean,
        pins.test_affinity_equals_average_token_affinity,
        pins.test_affinity_is_not_scaled_and_not_transposed,
        lambda: pins.test_topk_matches_subset_enumeration(7, True),
        pins.test_topk_duplicate_region_lower_index_first,
        lambda: pins.test_full_topk_is_dense_attention(2),
        lambda: pins.test_gather_equals_region_masked_dense((1, 12, 8, 6, 3, 4, 3)),
        pins.test_worked_example_by_hand,
        pins.test_region_permutation_equivariance,
        lambda: pins.test_brute_force_tiny(2, 2),
        lambda: pins.test_repeated_routes_attend_the_union(1),
    ]
    failures = 0
    with oracle.swapped_library(lib):
        for check in checks:
            try:
                check()
            except (AssertionError, ValueError):
                failures += 1
    assert failures > 0, f"no pin caught mutation {name}"


# The local context term's pins catch slips in its own function.
LCE_MUTATIONS = [
    ("lce_convolution_orientation", "int yy = y + i - 2;", "int yy = y - i + 2;"),
    ("lce_clamped_border", "if (yy < 0 || yy >= H) continue;",
     "if (yy < 0) yy = 0; if (yy >= H) yy = H - 1;"),
    ("lce_bias_dropped", "double acc = bias ? bias[c] : 0.0;", "double acc = 0.0;"),
    ("lce_taps_transposed", "acc += w[(size_t)c * 25 + i * 5 + j] *", "acc += w[(size_t)c * 25 + j * 5 + i] *"),
]


@pytest.mark.parametrize("name,old,new", LCE_MUTATIONS, ids=[m[0] for m in LCE_MUTATIONS])
def test_local_context_pins_catch_mutation(tmp_path, name, old, new):
    import test_oracle_lce as pins
    lib = build_variant(tmp_path, name, old, new)
    checks = [
        pins.test_matches_scipy_correlate2d_per_channel,
        pins.test_identity_kernel_returns_v,
        lambda: pins.test_single_tap_is_a_shift_with_zero_fill(1, -1),
        pins.test_constant_input_gives_kernel_sums,
        pins.test_bias_only,
    ]
    failures = 0
    with oracle.swapped_library(lib):
        for check in checks:
            try:
                check()
            except AssertionError:
                failures += 1
    assert failures > 0, f"no pin caught mutation {name}"


# The attention-gradient pins catch slips in the backward function.
BACKWARD_MUTATIONS = [
    ("bwd_missing_mean_term", "double ds = p[j] * (dp[j] - dsum);", "double ds = p[j] * dp[j];"),
    ("bwd_dk_unscaled", "dk[key_off[j] + c] += ds * q[qoff + c] * inv_sqrt_d;", "dk[key_off[j] + c] += ds * q[qoff + c];"),
    ("bwd_dv_from_ds", "dv[key_off[j] + c] += p[j] * g[qoff + c];", "dv[key_off[j] + c] += ds * g[qoff + c];"),
    ("bwd_repeats_counted_twice", "                    if (seen) continue;\n", ""),
]


@pytest.mark.parametrize("name,old,new", BACKWARD_MUTATIONS, ids=[m[0] for m in BACKWARD_MUTATIONS])
def test_backward_pins_catch_mutation(tmp_path, name, old, new):
    import test_oracle_backward as pins
    lib = build_variant(tmp_path, name, old, new)
    checks = [
        lambda: pins.test_gradients_match_finite_differences(1, 4, 4, 4, 1, 2, 2),
        pins.test_full_routing_is_dense_attention_gradient,
        pins.test_repeated_routes_count_once_like_a_masked_dense_attention,
    ]
    failures = 0
    with oracle.swapped_library(lib):
        for check in checks:
            try:
                check()
            except AssertionError:
                failures += 1
    assert failures > 0, f"no pin caught mutation {name}"


# The projection's pins catch slips in its own function.
QKV_MUTATIONS = [
    ("qkv_weight_transposed", "acc += w[(size_t)o * C + c] * xt[c];", "acc += w[(size_t)c * 3 * C + o] * xt[c];"),
    ("qkv_bias_dropped", "double acc = bias ? bias[o] : 0.0;", "double acc = 0.0;"),
    ("qkv_chunks_swapped", "double* dst = o < C ? q : (o < 2 * C ? k : v);",
     "double* dst = o < C ? k : (o < 2 * C ? q : v);"),
    ("qkv_channels_reversed", "dst[t * C + o % C] = acc;", "dst[t * C + (C - 1 - o % C)] = acc;"),
]


@pytest.mark.parametrize("name,old,new", QKV_MUTATIONS, ids=[m[0] for m in QKV_MUTATIONS])
def test_projection_pins_catch_mutation(tmp_path, name, old, new):
    import test_oracle_qkv as pins
    lib = build_variant(tmp_path, name, old, new)
    checks = [
        pins.test_block_identity_weights_give_scaled_copies,
        pins.test_bias_only_fills_each_chunk_with_its_bias,
        pins.test_permutation_rows_select_input_channels,
        lambda: pins.test_matches_numpy_matmul(True),
    ]
    failures = 0
    with oracle.swapped_library(lib):
        for check in checks:
            try:
                check()
            except AssertionError:
                failures += 1
    assert failures > 0, f"no pin caught mutation {name}"
