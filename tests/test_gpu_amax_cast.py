"""The one-pass amax + cast (fp8_amax_scale_cast) against fp8_amax followed by
fp8_scale_cast ("Training and inference of large language models using 8-bit
floating point", 제안 방법: the scale of each tensor from its own amax, then
the cast; "FP8-LM: Training FP8 Large Language Models", 提案手法 O1: mu).

The one-pass form casts with a predicted scale while it reduces the amax and
casts again only when the scale of that amax differs, so with a right and
with every kind of wrong prediction (another power of two, zero, NaN, a
value that is no power of two) its amax, scale, inverse and codes must be
those of the two-call form bit for bit.  The two-call form is held to the
oracle by test_gpu_parity.py; one case here checks the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_mixed_precision_tensor_b200 import fp8, synth

from test_gpu_parity import F32, scalar

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16, torch.float16]
FMTS = [fp8.FP8_E4M3, fp8.FP8_E5M2, fp8.FP8_F16S]


def _input(n, dtype, key, specials=False):
    x = synth.device_normal((n,), 3.0, key, torch.float32, "cuda")
    if n > 40 and specials:
        x[7] = float("inf")
        x[n - 3] = float("-inf")
    return x.to(dtype)


def _two_calls(x, fmt, margin, mu):
    a, s, inv = scalar(), scalar(), scalar()
    q = torch.empty(x.numel(), dtype=torch.int16 if fmt == fp8.FP8_F16S else torch.uint8, device="cuda")
    fp8.fp8_amax(x, a)
    fp8.fp8_scale_cast(x, fmt, a, margin, mu, s, inv, q)
    return a, s, inv, q


def _one_pass(x, fmt, margin, mu, pred):
    a, s, inv = scalar(), torch.full((1,), pred, **F32), scalar()
    q = torch.full((x.numel(),), 0x55, dtype=torch.int16 if fmt == fp8.FP8_F16S else torch.uint8, device="cuda")
    fp8.fp8_amax_scale_cast(x, fmt, a, margin, mu, s, inv, q)
    return a, s, inv, q


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n", [0, 1, 17, 4099, 65536 + 3, (1 << 20) + 5])
def test_one_pass_equals_amax_then_scale_cast(dtype, fmt, n):
    x = _input(n, dtype, 7 * n + fmt)
    for margin, mu in ((0, 1.0), (1, 2.0 ** 10 if fmt == fp8.FP8_E5M2 else 1.0)):
        ref = _two_calls(x, fmt, margin, mu)
        s = ref[1].item()
        for pred in (s, 2 * s, s / 4, 0.0, float("nan"), 3.0):
            got = _one_pass(x, fmt, margin, mu, pred)
            for name, r, g in zip(("amax", "scale", "inv", "codes"), ref, got):
                assert torch.equal(r.view(torch.int32) if r.dtype == torch.float32 else r,
                                   g.view(torch.int32) if g.dtype == torch.float32 else g), (name, margin, pred)
    assert fp8.fp8_get_status() == 0


def test_one_pass_with_specials_equals_the_two_calls():
    """inf elements (the amax is inf: the scale rule gives 2^0 and reports a
    non-finite amax) and a NaN (the amax is NaN): codes, scales and status as
    the two-call form's."""
    for poison in ("inf", "nan"):
        x = _input(4099, torch.bfloat16, 99, specials=True)
        if poison == "nan":
            x[100] = float("nan")
        for fmt in (fp8.FP8_E4M3, fp8.FP8_E5M2):
            ref = _two_calls(x, fmt, 0, 1.0)
            assert fp8.fp8_get_status() == 1  # FP8_STATUS_NONFINITE
            for pred in (1.0, 0.5):
                got = _one_pass(x, fmt, 0, 1.0, pred)
                assert fp8.fp8_get_status() == 1
                for r, g in zip(ref, got):
                    assert torch.equal(r.view(torch.int32) if r.dtype == torch.float32 else r,
                                       g.view(torch.int32) if g.dtype == torch.float32 else g)


def test_one_pass_against_the_oracle():
    n = 65536 + 11
    host = synth.normal_bf16((n,), 2.0, "amax-cast-oracle")
    x = torch.from_numpy(host.view(np.int16)).cuda().view(torch.bfloat16)
    for fmt, ofmt in ((fp8.FP8_E4M3, oracle.E4M3), (fp8.FP8_E5M2, oracle.E5M2)):
        a, s, inv, q = _one_pass(x, fmt, 1, 1.0, 1.0)
        amax = oracle.amax(host, oracle.DT_BF16)
        rc, s_ref = oracle.compute_scale(amax, ofmt, 1)
        assert a.item() == amax and s.item() == s_ref and inv.item() == 1.0 / s_ref
        assert np.array_equal(q.cpu().numpy(), oracle.cast(host, ofmt, s_ref, oracle.DT_BF16))


def test_one_pass_rejects_bad_arguments():
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(64, dtype=torch.uint8, device="cuda")
    a, s, inv = scalar(), scalar(), scalar()
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_amax_scale_cast(x, fp8.FP8_E4M3, a, 0, 3.0, s, inv, q)   # mu not a power of two
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_amax_scale_cast(x, 7, a, 0, 1.0, s, inv, q)              # no such format
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_amax_scale_cast(x[1:], fp8.FP8_E4M3, a, 0, 1.0, s, inv, q)  # unaligned
