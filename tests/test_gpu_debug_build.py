"""The debug build of the library (compiled with -DBRA_DEBUG) checks the output
index of every attention-kernel store against its buffer and reports a miss as
BRA_ERR_BOUNDS instead of writing.  This runs one case per attention kernel,
at the shapes each kernel covers, plus the attention with the local context
term and the tensor-core backward, through that build in a child process (the
package loads the build named by BRA_LIBRARY), and requires BRA_OK together
with parity against the oracle: no kernel computes an index outside its
output on these inputs."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, sys
sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
sys.path.insert(0, sys.argv[1])
import dynamic_sparse_attention_bra_b200 as bra
assert bra.library_path.endswith("libbra_b200_debug.so"), bra.library_path
import bra_inputs as bi
from test_gpu_parity import check_case
cases = [
    ("slice", (2, 14, 14, 256, 8, 7, 16, "bf16")),
    ("warp", (2, 28, 28, 128, 4, 7, 4, "bf16")),
    ("warp", (3, 28, 28, 96, 3, 7, 4, "bf16")),
    ("flash", (1, 64, 64, 64, 2, 4, 2, "bf16")),
    ("stack", (4, 56, 56, 64, 2, 7, 1, "bf16")),
    ("stack", (2, 28, 28, 128, 4, 7, 4, "bf16")),
    ("tiled", (1, 32, 32, 64, 2, 2, 2, "bf16")),
    ("tiled", (2, 24, 24, 64, 2, 4, 3, "bf16")),
    ("simt", (2, 24, 24, 64, 2, 4, 3, "f32")),
]
for kernel, dims in cases:
    os.environ["BRA_ATTEND_KERNEL"] = kernel
    err, rep = check_case(bi.BraShape(*dims), 77)  # asserts BRA_OK and parity
    print(kernel, dims, "ok", f"{err:.2e}")
os.environ.pop("BRA_ATTEND_KERNEL")
# the local context term in the stack kernel's epilogue (asserts BRA_OK and parity)
from test_gpu_forward_lce import check_forward_lce
check_forward_lce(bi.BraShape(2, 56, 56, 64, 2, 7, 1, "bf16"), 78, "debug build [fused lce]")
print("fused lce", "ok")
# the tensor-core backward (asserts BRA_OK and parity within its bound)
import test_gpu_backward as tb
class Env:
    def setenv(self, k, v): os.environ[k] = v
    def delenv(self, k, raising=True): os.environ.pop(k, None)
for dims in ((2, 56, 56, 64, 2, 7, 1), (2, 28, 28, 128, 4, 7, 4)):
    shape = bi.BraShape(*dims, "bf16")
    status, got, ref, (inp, idx, g64) = tb.run(shape, 79, "mma", Env())
    assert status == bra.BRA_OK, status
    tb.check(shape, got, ref, "mma", "debug build", tb.mma_bounds(shape, inp, idx, g64))
    print("backward mma", dims, "ok")
"""


def test_debug_build_reports_no_out_of_bounds_index():
    lib = os.path.join(ROOT, "dynamic_sparse_attention_bra_b200", "libbra_b200_debug.so")
    assert os.path.exists(lib), "the debug build is made by __graft_entry__.build()"
    env = dict(os.environ, BRA_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert r.stdout.count(" ok") == 12, r.stdout
