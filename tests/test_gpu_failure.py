"""Failure detection without a GPU fault: a bounded wait that runs out is
recorded as BRA_ERR_TIMEOUT in the workspace status block, the host reads it,
and the same CUDA context keeps working (the next forward is correct)."""
import pytest

import bra_inputs as bi
from gpu_helpers import run_forward

pytestmark = pytest.mark.gpu


def setup():
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    s = bra.shape_for(1, 16, 16, 64, 2, 4, 2, "bf16")
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    return bra, s, ws


def test_wait_on_a_barrier_nobody_arrives_at_times_out():
    bra, s, ws = setup()
    bra.bra_selftest_bounded_wait(s, ws, 1000, arrive=False)
    assert bra.bra_device_status(s, ws) == bra.BRA_ERR_TIMEOUT
    assert bra.bra_device_status(s, ws) == bra.BRA_OK  # reading clears it


def test_satisfied_wait_records_nothing():
    bra, s, ws = setup()
    bra.bra_selftest_bounded_wait(s, ws, 1000, arrive=True)
    assert bra.bra_device_status(s, ws) == bra.BRA_OK


def test_context_usable_after_a_timeout():
    from test_gpu_parity import check_case
    bra, s, ws = setup()
    bra.bra_selftest_bounded_wait(s, ws, 1000, arrive=False)
    assert bra.bra_device_status(s, ws) == bra.BRA_ERR_TIMEOUT
    check_case(bi.BraShape(2, 24, 24, 64, 2, 4, 3, "bf16"), 31)
