"""The library's branch-free FP8 encoder, exhaustively.

Every FP8 code the library writes (casts, the sum of codes, Adam's first
moment and E4M3 weight copy) comes from one encoder: the saturating hardware
conversion of two binary32 values, with NaN codes made 0x7F by byte-wise
SIMD compares and no per-value test.  It must give exactly the codes of the
same conversion with an explicit test for inf and NaN (+-inf -> +-max, NaN
-> 0x7F: the definition the oracle's cast follows, "Training and inference
of large language models using 8-bit floating point", 제안 방법) -- checked
here on all 2^32 binary32 values, in each lane, for E4M3 and E5M2.
"""
import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
def test_encoder_equals_the_checked_encoder_on_every_binary32(fmt):
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    fp8.fp8_selftest_encode(fmt, 0, 1 << 32, bad, first)
    assert bad.item() == 0, (bad.item(), hex(first.item() & 0xFFFFFFFF))


def test_encode_selftest_rejects_bad_arguments():
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(1, dtype=torch.int32, device="cuda")
    for fmt, lo, hi in ((fp8.FP8_F16S, 0, 16), (fp8.FP8_E4M3, 16, 16), (fp8.FP8_E5M2, 0, (1 << 32) + 1)):
        with pytest.raises(fp8.FP8Error):
            fp8.fp8_selftest_encode(fmt, lo, hi, bad, first)
