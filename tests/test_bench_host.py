"""Host-side pieces of bench.py that the GPU line rests on: the minimal-byte
counts behind the rooflines, the options that pick what one run times, and
the rule that keys each recorded DRAM-traffic figure to the kernel's code."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import bra_inputs as bi  # noqa: E402


def test_stage1_byte_counts():
    """Counted by hand for B64 56x56 C64, 2 heads, S7, topk 1, bf16."""
    shape = bi.WORKLOADS["stage1"][0]
    cnt = bench.byte_counts(shape)
    tokens = 64 * 56 * 56
    assert cnt["map"] == tokens * 64 * 2 == 25_690_112
    assert cnt["idx"] == 64 * 2 * 49 * 1 * 4
    assert cnt["attend"] == 4 * 25_690_112 + 25_088 == 102_785_536  # Q, K, V read, O written, I^r
    # gradients: Q, K, V, dO and I^r read; dQ, dK, dV written in fp32
    assert cnt["backward"] == 4 * 25_690_112 + 25_088 + 3 * tokens * 64 * 4 == 256_926_208


@pytest.mark.parametrize("name", ["stage2", "stage3", "highres", "tiny"])
def test_backward_bytes_are_inputs_plus_fp32_gradients(name):
    shape = bi.WORKLOADS[name][0]
    cnt = bench.byte_counts(shape)
    es = 2 if shape.dtype == "bf16" else 4
    grads = 3 * shape.B * shape.H * shape.W * shape.C * 4
    assert cnt["backward"] == 4 * shape.B * shape.H * shape.W * shape.C * es + cnt["idx"] + grads


def test_extras_and_per_workload_options():
    a = bench.parse([])
    assert a.extras.split(",") == ["backward", "lce"]
    assert a.per_workload.split(",") == ["stage2", "stage3", "highres"]
    a = bench.parse(["--extras", "none", "--per-workload", "none"])
    assert [e for e in a.extras.split(",") if e in ("backward", "lce")] == []
    assert [w for w in a.per_workload.split(",") if w in bi.WORKLOADS] == []


def test_traffic_key_ignores_comments_only():
    code = "int a = 1;\n__device__ void f() { a += 2; }\n"
    commented = "// header comment\nint a = 1;  // one\n/* block\n comment */\n__device__ void f() { a += 2; }\n\n"
    assert bench._code_only(code) == bench._code_only(commented)
    assert bench._code_only(code) != bench._code_only(code.replace("2", "3"))


def test_traffic_records_name_existing_kernel_files():
    csrc = os.path.join(ROOT, "dynamic_sparse_attention_bra_b200", "csrc")
    for name in bench.TRAFFIC_RECORDS:
        assert os.path.exists(os.path.join(csrc, name)), name
    for workload, name in bench.KERNEL_FILE.items():
        assert workload in bi.WORKLOADS and os.path.exists(os.path.join(csrc, name))
