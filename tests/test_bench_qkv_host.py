"""Host side of the projection workloads: the seeded linear-layer inputs and
the benchmark's reference arm when every step starts from the feature map."""
import json

import numpy as np
import pytest

import bench
import bra_inputs as bi


def test_projection_inputs_are_seeded_and_bounded():
    shape = bi.BraShape(2, 16, 16, 64, 2, 4, 2, "bf16")
    a = bi.make_projection_inputs(shape, 3)
    b = bi.make_projection_inputs(shape, 3)
    c = bi.make_projection_inputs(shape, 4)
    assert (a.x_store == b.x_store).all() and (a.w_store == b.w_store).all() and (a.b_store == b.b_store).all()
    assert not (a.w_store == c.w_store).all()
    assert a.w_f64.shape == (192, 64) and a.b_f64.shape == (192,) and a.x_f64.shape == (2, 16, 16, 64)
    bound = 1.0 / np.sqrt(64)
    assert np.abs(a.w_f64).max() <= bound and np.abs(a.b_f64).max() <= bound
    # bf16 storage: the widened values survive a round trip through bf16 unchanged
    np.testing.assert_array_equal(bi.f32_to_bf16_bits(a.w_f64.astype(np.float32)), a.w_store)
    # X is its own stream, not one of Q, K, V
    q = bi.make_inputs(shape, 3).q_store
    assert not (q == a.x_store).all()


def test_projection_inputs_are_bf16_only():
    with pytest.raises(ValueError):
        bi.make_projection_inputs(bi.BraShape(1, 16, 16, 32, 1, 4, 2, "f32"), 0)


def test_projection_byte_count_adds_up():
    shape = bi.WORKLOADS["stage1"][0]
    cnt = bench.byte_counts(shape)
    # X read and Q, K, V written are four maps; the means and the layer are small
    assert 4 * cnt["map"] < cnt["qkv"] < 4 * cnt["map"] + 2 * 2**20
    assert cnt["path_min_qkv"] == 2 * cnt["map"] + cnt["idx"]


def test_reference_arm_from_feature_map(capsys):
    args = bench.parse(["--impl", "reference", "--qkv", "--workload", "detection", "--steps", "1",
                        "--warmup", "0"])
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["from_feature_map"] is True
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
