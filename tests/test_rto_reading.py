"""Pins of the round-to-odd bfloat16 GEMM output (FP8_DT_BF16_RTO).

The wgrad may store dW as bfloat16 rounded to odd instead of float32 because
the FP8 gradient cast that follows cannot tell the two apart: bfloat16 keeps
8 significant bits, at least 2 more than E5M2 (3) or E4M3 (4), so rounding
to nearest even from the round-to-odd value lands where rounding the float32
value would, and every power-of-two scale threshold (fmt_max * 2^-e) is a
bfloat16 value that round-to-odd never crosses.  These checks run the
oracle's own cast, scale rule and counters on float32 values and on their
round-to-odd bfloat16 images, with round-to-odd written here from its
definition, and require identical codes, scales and counts.
"""
import numpy as np
import pytest

import oracle
from fp8_mixed_precision_tensor_b200 import synth

DT_BF16 = 1


def rto_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bits rounded to odd: keep the top 16 bits and set
    the last one when any dropped bit was set."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    hi = (u >> 16).astype(np.uint16)
    return hi | ((u & 0xFFFF) != 0).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _adversarial(fmt: int, n_random: int, seed: str) -> np.ndarray:
    """Values on, just beside and between every rounding midpoint and code of
    the format (scaled by a few powers of two), plus log-uniform randoms."""
    table = oracle.decode_table(fmt)
    finite = np.unique(np.abs(table[np.isfinite(table)]))
    mids = (finite[:-1] + finite[1:]) / 2.0
    pts = np.concatenate([finite, mids]).astype(np.float32)
    f32 = []
    for p in pts:
        for k in (-3, -2, -1, 1, 2, 3, 40, 1000):
            f32.append(np.nextafter(p, np.float32(np.inf) if k > 0 else np.float32(0)) if abs(k) < 4 else p)
            # offsets of a few float32 ulps and of fractions of a bfloat16 ulp around the point
            f32.append(np.float32(p) * np.float32(1.0 + k * 2.0 ** -20))
    base = np.array(f32 + list(pts), dtype=np.float32)
    rng = synth.rng("rto-pin", seed)
    rnd = (rng.choice([-1.0, 1.0], n_random) * np.exp(rng.uniform(-14.0, 14.0, n_random))).astype(np.float32)
    both = np.concatenate([base, -base, rnd])
    return both[np.isfinite(both)]


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("scale_exp", [-12, -4, 0, 3, 9])
def test_fp8_cast_of_rto_bf16_equals_cast_of_float32(fmt, scale_exp):
    x = _adversarial(fmt, 200000, f"{fmt}-{scale_exp}") * np.float32(2.0 ** -scale_exp)
    x = x[np.isfinite(x)]
    s = 2.0 ** scale_exp
    ref, ref_counts = oracle.cast_counts(x, fmt, s)
    bits = rto_bf16_bits(x)
    got, got_counts = oracle.cast_counts(bits, fmt, s, dtype=DT_BF16)
    bad = ref != got
    assert not bad.any(), (x[bad][:5], ref[bad][:5], got[bad][:5])
    assert ref_counts == got_counts


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_scale_of_rto_amax_equals_scale_of_float32_amax(fmt):
    """Every threshold fmt_max * 2^-e and its neighbours: the scale rule gives
    the same exponent for an amax and for its round-to-odd image."""
    fmax = oracle.fmt_max(fmt)
    vals = []
    for e in range(-30, 31):
        t = np.float32(fmax * 2.0 ** -e)
        vals += [t, np.nextafter(t, np.float32(np.inf)), np.nextafter(t, np.float32(0)),
                 t * np.float32(1 + 2.0 ** -9), t * np.float32(1 - 2.0 ** -9)]
    vals += list(_adversarial(fmt, 20000, f"amax-{fmt}"))
    for margin in (0, 1):
        for a in vals:
            a = np.float32(abs(a))
            if a == 0:
                continue
            r = bf16_to_f32(rto_bf16_bits(np.array([a])))[0]
            assert oracle.compute_scale(float(a), fmt, margin) == oracle.compute_scale(float(r), fmt, margin), \
                (a, r, margin)


def test_rto_is_monotone_and_keeps_specials():
    x = np.array([0.0, -0.0, np.inf, -np.inf, 1.0, 1.0 + 2.0 ** -20, -(1.0 + 2.0 ** -20)], dtype=np.float32)
    b = rto_bf16_bits(x)
    assert list(b[:6]) == [0x0000, 0x8000, 0x7F80, 0xFF80, 0x3F80, 0x3F81]
    nan = np.array([0x7F800001], dtype=np.uint32).view(np.float32)
    assert np.isnan(bf16_to_f32(rto_bf16_bits(nan)))[0]
    y = np.sort(_adversarial(oracle.E5M2, 5000, "mono"))
    r = bf16_to_f32(rto_bf16_bits(y))
    assert np.all(np.diff(r) >= 0)


def test_round_to_nearest_or_truncation_would_not_do():
    """The same values discriminate: rounding to nearest even, or truncating,
    to bfloat16 first changes thousands of codes (double rounding)."""
    import torch

    x = _adversarial(oracle.E5M2, 200000, "discriminate")
    ref = oracle.cast(x, oracle.E5M2, 1.0)
    rn = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    trunc = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.count_nonzero(oracle.cast(rn, oracle.E5M2, 1.0, dtype=DT_BF16) != ref) > 100
    assert np.count_nonzero(oracle.cast(trunc, oracle.E5M2, 1.0, dtype=DT_BF16) != ref) > 100
    assert np.count_nonzero(oracle.cast(rto_bf16_bits(x), oracle.E5M2, 1.0, dtype=DT_BF16) != ref) == 0
