"""Failure detection without a GPU fault: the library's pipeline waits are
bounded, and a wait that runs out ends with a status the host reads, leaving
the context usable.  The wait is made to run out on a barrier that nothing
arrives at (nothing faults, traps or hangs)."""
import numpy as np
import torch

import pytest

from fp8_mixed_precision_tensor_b200 import fp8

pytestmark = pytest.mark.gpu


def test_bounded_pipeline_wait_times_out_into_a_status():
    """The GEMM pipeline's barrier wait, run on a barrier nothing arrives at
    with a 2 ms limit, ends by itself and raises FP8_STATUS_TIMEOUT; the
    status reads back once and is cleared, and the context stays usable (a
    GEMM right after gives the exact product of all-ones operands)."""
    assert fp8.fp8_get_status() == 0
    fp8.fp8_selftest_wait_timeout(2000)
    assert fp8.fp8_get_status() == fp8.FP8_STATUS_TIMEOUT
    assert fp8.fp8_get_status() == 0
    # E4M3 code 0x38 = 1.0: every output of a 32x32x32 product of ones is 32
    a = torch.full((32, 32), 0x38, dtype=torch.uint8, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    y = torch.zeros((32, 32), dtype=torch.float32, device="cuda")
    fp8.fp8_linear_fwd(a, one, a, one, y)
    assert np.all(y.cpu().numpy() == 32.0) and fp8.fp8_get_status() == 0
