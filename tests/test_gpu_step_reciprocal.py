"""The Adam step's correctly rounded reciprocal, exhaustively.

The update computes RN(1 / (sqrt(v_hat) + eps)) with its own branch-free
reciprocal (the MUFU approximation and one Newton-Raphson correction whose
residual is taken in a fused multiply-add) instead of CUDA's __frcp_rn.  The
two must agree bit for bit on every binary32 argument the step can give it --
[2^-39, 2^66], the range of sqrt(v_hat) + eps for 2^-39 <= eps <= 2^64, and
+inf -- so the step's results are those of the correctly rounded operation.
"""
import struct

import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8

pytestmark = pytest.mark.gpu


def _sweep(lo, hi):
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    fp8.fp8_selftest_step_reciprocal(lo, hi, bad, first)
    return bad.item(), first.item() & 0xFFFFFFFF


def bits(x):
    return struct.unpack("<I", struct.pack("<f", x))[0]


def test_step_reciprocal_equals_the_correctly_rounded_one_on_its_range():
    nbad, first = _sweep(bits(2.0 ** -39), bits(2.0 ** 66) + 1)
    assert nbad == 0, (nbad, hex(first))
    nbad, first = _sweep(bits(float("inf")), bits(float("inf")) + 1)
    assert nbad == 0


def test_selftest_finds_a_difference_where_there_is_one():
    """Outside the step's range the reciprocal of a large argument is a
    binary32 subnormal, which the flush-to-zero approximation does not give:
    the self-test reports those arguments, so it does compare."""
    nbad, first = _sweep(bits(2.0 ** 127), bits(2.0 ** 127) + 4096)
    assert nbad == 4096 and first == bits(2.0 ** 127)


def test_selftest_rejects_bad_arguments():
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(1, dtype=torch.int32, device="cuda")
    for lo, hi in ((16, 16), (0, (1 << 32) + 1)):
        with pytest.raises(fp8.FP8Error):
            fp8.fp8_selftest_step_reciprocal(lo, hi, bad, first)
