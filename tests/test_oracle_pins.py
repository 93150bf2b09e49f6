"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each check compares the oracle with something it does not share code with:
the format definitions (golden fixture), brute force over all codes, closed
forms of the scale rule, independent library routines (torch's float8 and
numpy's float16 conversions, numpy matmul, torch.optim.Adam) and invariants.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_mixed_precision_tensor_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ofp8_points.txt")
FMTS = {"E4M3": oracle.E4M3, "E5M2": oracle.E5M2}
TORCH_FP8 = {oracle.E4M3: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}
TOP = {oracle.E4M3: 0x7E, oracle.E5M2: 0x7B}


def _parse(v):
    return {"nan": math.nan, "inf": math.inf, "-inf": -math.inf, "-0": -0.0}.get(v, None) if v in (
        "nan", "inf", "-inf", "-0") else float(v)


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        fmt, code, val = line.split()
        rows.append((fmt, int(code, 16), _parse(val)))
    return rows


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


# ---------------------------------------------------------------- formats
def test_golden_format_points():
    for fmt, code, val in _golden():
        got = oracle.f16_decode(code) if fmt == "F16" else oracle.decode(FMTS[fmt], code)
        assert _same(got, val), (fmt, hex(code), got, val)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_decode_table_matches_torch_float8(fmt):
    ours = oracle.decode_table(fmt)
    ref = torch.arange(256, dtype=torch.uint8).view(TORCH_FP8[fmt]).double().numpy()
    for c in range(256):
        assert _same(ours[c], ref[c]), (fmt, hex(c), ours[c], ref[c])


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_finite_codes_monotone_and_max(fmt):
    t = oracle.decode_table(fmt)
    pos = t[: TOP[fmt] + 1]
    assert np.all(np.diff(pos) > 0)
    assert oracle.fmt_max(fmt) == {oracle.E4M3: 448.0, oracle.E5M2: 57344.0}[fmt]
    # negative half mirrors the positive half
    for c in range(128):
        a, b = t[c], t[c | 0x80]
        assert (math.isnan(a) and math.isnan(b)) or a == -b


def test_f16_decode_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 7):  # every 7th pattern (all classes are hit)
        assert _same(oracle.f16_decode(b), ref[b]), hex(b)
    for b in (0x0000, 0x8000, 0x0001, 0x03FF, 0x0400, 0x7BFF, 0x7C00, 0xFC00, 0x7E00):
        assert _same(oracle.f16_decode(b), ref[b]), hex(b)


# ---------------------------------------------------------------- encode
@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_roundtrip_all_codes(fmt):
    for c in range(256):
        v = oracle.decode(fmt, c)
        e = oracle.encode(fmt, v)
        if math.isnan(v):
            assert e in (0x7F, 0xFF)
        elif math.isinf(v):  # E5M2 inf saturates to max (satfinite reading)
            assert e == (c & 0x80) | TOP[fmt]
        else:
            assert e == c, (fmt, hex(c), hex(e))


def _brute_nearest(fmt, y):
    """argmin over all finite codes of |dec(c) - y|, ties to even mantissa; saturating."""
    t = oracle.decode_table(fmt)
    best, bestd = None, None
    for c in range(256):
        v = t[c]
        if not math.isfinite(v):
            continue
        if math.copysign(1, v) != math.copysign(1, y) and v != 0:
            continue
        if (c & 0x80) != (0x80 if math.copysign(1, y) < 0 else 0):
            continue
        d = abs(v - y)
        if bestd is None or d < bestd or (d == bestd and (c & 1) == 0):
            best, bestd = c, d
    return best


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_brute_force_random_and_midpoints(fmt):
    t = oracle.decode_table(fmt)
    pos = t[: TOP[fmt] + 1]
    mids = list((pos[:-1] + pos[1:]) / 2)
    mids += [pos[-1] * 1.0 + (pos[-1] - pos[-2]) / 2]  # midpoint above max -> saturates
    g = synth.rng("pin", "encode", fmt)
    ys = list(g.uniform(0, pos[-1] * 1.2, 400)) + list(np.exp(g.uniform(-14, 0, 400)) * pos[-1])
    ys += mids + [pos[-1] * 10, 0.0]
    for y in ys:
        for s in (1.0, -1.0):
            assert oracle.encode(fmt, s * y) == _brute_nearest(fmt, s * y), (fmt, s * y)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_matches_torch_in_range(fmt):
    g = synth.rng("pin", "encode-torch", fmt)
    mx = oracle.fmt_max(fmt)
    y = np.concatenate([g.uniform(-mx, mx, 20000), np.exp(g.uniform(-25, math.log(mx), 20000))
                        * np.where(g.random(20000) < 0.5, -1, 1)]).astype(np.float32)
    y = y[np.abs(y) <= mx]
    ref = torch.from_numpy(y).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    ours = oracle.cast(y, fmt, 1.0)
    assert np.array_equal(ours, ref)


def test_encode_saturation_and_specials():
    for fmt in (oracle.E4M3, oracle.E5M2):
        mx = oracle.fmt_max(fmt)
        for y in (mx * 1.01, mx * 2, 1e30, math.inf):
            assert oracle.encode(fmt, y) == TOP[fmt]
            assert oracle.encode(fmt, -y) == 0x80 | TOP[fmt]
        assert oracle.encode(fmt, -0.0) == 0x80
        assert oracle.encode(fmt, 0.0) == 0x00
        assert oracle.encode(fmt, 1e-30) == 0x00
        assert oracle.encode(fmt, -1e-30) == 0x80
    assert oracle.encode(oracle.E4M3, 464.0) == 0x7E  # tie above max -> max
    assert oracle.encode(oracle.E5M2, 61440.0) == 0x7B


def test_f16_encode_matches_numpy():
    g = synth.rng("pin", "f16")
    y = np.concatenate([g.normal(0, 1, 20000), np.exp(g.uniform(-20, 11, 20000)),
                        g.uniform(65000, 65519.9, 100)])
    ref = y.astype(np.float16).view(np.uint16)
    for a, r in zip(y, ref):
        assert oracle.f16_encode(a) == r, a
    # exact midpoints between consecutive halves round to even
    h = np.arange(0x3C00, 0x3C40, dtype=np.uint16).view(np.float16).astype(np.float64)
    for lo, hi in zip(h[:-1], h[1:]):
        mid = (lo + hi) / 2
        assert oracle.f16_encode(mid) == np.float64(mid).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------------- amax
def test_amax_matches_numpy():
    x = synth.normal_f32((10007,), 3.0, "pin", "amax")
    assert oracle.amax(x) == float(np.max(np.abs(x)))
    b = synth.lognormal_outliers_bf16(50001, "pin", "amax-bf16")
    ref = float(np.max(np.abs(synth.bf16_bits_to_f32(b))))
    assert oracle.amax(b, oracle.DT_BF16) == ref
    assert oracle.amax(b, oracle.DT_BF16, parallel=True) == ref
    h = (x / 8).astype(np.float16)
    assert oracle.amax(h.view(np.uint16), oracle.DT_F16) == float(np.max(np.abs(h.astype(np.float64))))


def test_amax_specials():
    x = np.array([1.0, -3.0, 2.0], np.float32)
    assert oracle.amax(x) == 3.0
    x2 = np.array([1.0, -np.inf, 2.0], np.float32)
    assert oracle.amax(x2) == math.inf
    x3 = np.array([1.0, np.nan, -np.inf], np.float32)
    assert math.isnan(oracle.amax(x3))
    assert oracle.amax(np.array([-0.0, 0.0], np.float32)) == 0.0
    assert oracle.amax(np.zeros(0, np.float32)) == 0.0


# ---------------------------------------------------------------- scale rule
def _brute_exponent(amax, fmt_max):
    best = None
    for e in range(-400, 400):
        if math.ldexp(amax, e) <= fmt_max:
            best = e
    return best


def test_scale_closed_forms():
    E4, E5 = oracle.E4M3, oracle.E5M2
    assert oracle.compute_scale(448.0, E4, 0) == (0, 1.0)
    assert oracle.compute_scale(448.0 * (1 + 2 ** -23), E4, 0) == (0, 0.5)
    assert oracle.compute_scale(1.0, E4, 0) == (0, 256.0)
    assert oracle.compute_scale(1.0, E5, 0) == (0, 32768.0)
    assert oracle.compute_scale(1.0, E4, 1) == (0, 128.0)
    assert oracle.compute_scale(57344.0, E5, 0) == (0, 1.0)
    assert oracle.compute_scale(65504.0, oracle.F16, 0) == (0, 1.0)
    assert oracle.compute_scale(0.0, E4, 3) == (0, 1.0)
    rc, s = oracle.compute_scale(math.inf, E4, 0)
    assert rc == oracle.ERR_NONFINITE and s == 1.0
    rc, s = oracle.compute_scale(math.nan, E5, 0)
    assert rc == oracle.ERR_NONFINITE and s == 1.0
    # clamping keeps s and 1/s normal binary32
    assert oracle.compute_scale(1e-45, E4, 0) == (0, 2.0 ** 126)
    assert oracle.compute_scale(1e38, E4, 10) == (0, 2.0 ** -126)
    # total multiplier mu * s_g = 2^103 * 2^32 is clamped to 2^126 as well
    assert oracle.compute_scale(1e-38, E4, 0, mu=2.0 ** 32) == (0, 2.0 ** 126)


def test_scale_rule_brute_force():
    g = synth.rng("pin", "scale")
    vals = list(np.exp(g.uniform(-80, 80, 2000)))
    for fmt in (oracle.E4M3, oracle.E5M2, oracle.F16):
        mx = oracle.fmt_max(fmt)
        vals_f = vals + [mx, mx * 2, mx / 2, math.nextafter(mx, 0), math.nextafter(mx, 10 * mx),
                         mx * 2 ** -20, np.float32(mx * 3 / 7)]
        for a in vals_f:
            a = float(np.float32(a))
            e = _brute_exponent(a, mx)
            assert oracle.floor_log2_ratio(a, mx) == e, (fmt, a)
            for margin in (0, 1, 3):
                rc, s = oracle.compute_scale(a, fmt, margin)
                k = max(-126, min(126, e - margin))
                assert rc == 0 and s == 2.0 ** k


def test_scale_invariants_and_mu():
    g = synth.rng("pin", "scale-inv")
    for fmt in (oracle.E4M3, oracle.E5M2):
        mx = oracle.fmt_max(fmt)
        for _ in range(300):
            a = float(np.float32(math.exp(g.uniform(-30, 30))))
            for margin in (0, 1, 2):
                _, s = oracle.compute_scale(a, fmt, margin)
                assert a * s <= mx / 2 ** margin
                if margin == 0:
                    assert a * s > mx / 2
            # mu invariance for powers of two: the total scale does not depend on mu
            # (the combined multiplier is clamped to normal binary32 like any scale)
            base = oracle.compute_scale(a, fmt, 0, mu=1.0)[1]
            for mu in (2.0 ** 10, 2.0 ** -4, 2.0 ** 3):
                assert oracle.compute_scale(a, fmt, 0, mu=mu)[1] == base


# ---------------------------------------------------------------- cast
def test_cast_matches_torch_and_never_saturates():
    b = synth.lognormal_outliers_bf16(1 << 16, "pin", "cast")
    x = synth.bf16_bits_to_f32(b)
    a = oracle.amax(b, oracle.DT_BF16)
    for fmt in (oracle.E4M3, oracle.E5M2):
        for margin in (0, 1):
            _, s = oracle.compute_scale(a, fmt, margin)
            q = oracle.cast(b, fmt, s, oracle.DT_BF16)
            y = torch.from_numpy(x.astype(np.float64) * s)
            assert float(y.abs().max()) <= oracle.fmt_max(fmt)
            ref = y.float().to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
            assert np.array_equal(q, ref)
            # represented values dec(q)/s recover x within half a code step
            dec = oracle.decode_table(fmt)[q] / s
            assert np.all(np.isfinite(dec))


def test_cast_mu_invariance_codes_identical():
    g = synth.normal_f32((4096,), 1e-3, "pin", "mu")
    a = oracle.amax(g)
    base = None
    for mu in (1.0, 2.0 ** 10, 2.0 ** -4):
        _, st = oracle.compute_scale(a, oracle.E5M2, 0, mu=mu)
        q = oracle.cast(g, oracle.E5M2, st)
        if base is None:
            base = q
        assert np.array_equal(q, base)


def test_cast_f16_matches_numpy():
    x = synth.normal_f32((5000,), 0.02, "pin", "castf16")
    _, s = oracle.compute_scale(oracle.amax(x), oracle.F16, 0)
    q = oracle.cast(x, oracle.F16, s)
    ref = (x.astype(np.float64) * s).astype(np.float16).view(np.uint16)
    assert np.array_equal(q, ref)


# ---------------------------------------------------------------- GEMMs
def _torch_dec(codes, fmt):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(TORCH_FP8[fmt]).double().numpy()


def _codes(shape, fmt, *key):
    """Random finite codes of a format."""
    g = synth.rng(*key)
    c = g.integers(0, 256, size=shape).astype(np.uint8)
    bad = ~np.isfinite(oracle.decode_table(fmt)[c])
    c[bad] = 0x38 if fmt == oracle.E4M3 else 0x3C
    return c


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 7), (16, 48, 32), (128, 128, 128)])
def test_gemm_fwd_dgrad_wgrad_vs_numpy(shape):
    M, N, K = shape
    xq = _codes((M, K), oracle.E4M3, "pin", "gx", shape)
    wq = _codes((N, K), oracle.E4M3, "pin", "gw", shape)
    dyq = _codes((M, N), oracle.E5M2, "pin", "gdy", shape)
    sx, sw, sdy = 2.0 ** -3, 2.0 ** 5, 2.0 ** 12
    X, W, DY = _torch_dec(xq, 0) / sx, _torch_dec(wq, 0) / sw, _torch_dec(dyq, 1) / sdy
    bias = synth.normal_f32((N,), 1.0, "pin", "bias", shape).astype(np.float64)
    Y, Yabs = oracle.linear_fwd(xq, 1 / sx, wq, 1 / sw, M, N, K, bias=bias)
    np.testing.assert_allclose(Y, X @ W.T + bias, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(Yabs, np.abs(X) @ np.abs(W).T, rtol=1e-12)
    dX, _ = oracle.linear_dgrad(dyq, 1 / sdy, wq, 1 / sw, M, N, K)
    np.testing.assert_allclose(dX, DY @ W, rtol=1e-12, atol=1e-300)
    dW, _ = oracle.linear_wgrad(dyq, 1 / sdy, xq, 1 / sx, M, N, K)
    np.testing.assert_allclose(dW, DY.T @ X, rtol=1e-12, atol=1e-300)
    assert dX.shape == (M, K) and dW.shape == (N, K)


def test_gemm_exact_integer_case_and_identity():
    # codes for +-1 and +-2 only: every product and partial sum is an exact small integer
    M = N = K = 64
    g = synth.rng("pin", "gint")
    pick = np.array([0x38, 0xB8, 0x40, 0xC0], np.uint8)  # E4M3 +1, -1, +2, -2
    xq, wq = pick[g.integers(0, 4, (M, K))], pick[g.integers(0, 4, (N, K))]
    Y, _ = oracle.linear_fwd(xq, 1.0, wq, 1.0, M, N, K)
    Xi = np.select([xq == 0x38, xq == 0xB8, xq == 0x40], [1, -1, 2], -2).astype(np.int64)
    Wi = np.select([wq == 0x38, wq == 0xB8, wq == 0x40], [1, -1, 2], -2).astype(np.int64)
    assert np.array_equal(Y, (Xi @ Wi.T).astype(np.float64))
    # identity W returns the dequantised X
    eye = np.where(np.eye(K, dtype=bool), np.uint8(0x38), np.uint8(0x00))
    xq2 = _codes((M, K), oracle.E4M3, "pin", "gid")
    Y2, _ = oracle.linear_fwd(xq2, 0.25, eye, 1.0, M, K, K)
    np.testing.assert_array_equal(Y2, oracle.decode_table(0)[xq2] * 0.25)


def test_gemm_sampled_equals_full():
    M, N, K = 40, 24, 56
    xq = _codes((M, K), 0, "pin", "sx")
    wq = _codes((N, K), 0, "pin", "sw")
    Y, Ya = oracle.linear_fwd(xq, 0.5, wq, 2.0, M, N, K)
    g = synth.rng("pin", "ss")
    r, c = g.integers(0, M, 50), g.integers(0, N, 50)
    Ys, Yas = oracle.linear_fwd(xq, 0.5, wq, 2.0, M, N, K, samples=(r, c))
    np.testing.assert_array_equal(Ys, Y[r, c])
    np.testing.assert_array_equal(Yas, Ya[r, c])


# ---------------------------------------------------------------- Adam
HP = dict(lr=1e-4, beta1=0.9, beta2=0.95, eps=1e-8)


def _torch_adam(g, m0, v0, w0, t, lr, beta1, beta2, eps):
    p = torch.nn.Parameter(torch.from_numpy(w0.copy()))
    opt = torch.optim.Adam([p], lr=lr, betas=(beta1, beta2), eps=eps, foreach=False)
    p.grad = torch.from_numpy(g.copy())
    opt.state[p] = {"step": torch.tensor(float(t - 1), dtype=torch.float64),
                    "exp_avg": torch.from_numpy(m0.copy()), "exp_avg_sq": torch.from_numpy(v0.copy())}
    opt.step()
    st = opt.state[p]
    return st["exp_avg"].numpy(), st["exp_avg_sq"].numpy(), p.detach().numpy()


@pytest.mark.parametrize("t", [1, 2, 7])
def test_adam_update_matches_torch_optim(t):
    n = 333
    g = synth.normal_f32((n,), 1e-3, "pin", "adam", t).astype(np.float64)
    m0 = synth.normal_f32((n,), 1e-3, "pin", "m0", t).astype(np.float64) * (t > 1)
    v0 = np.abs(synth.normal_f32((n,), 1e-6, "pin", "v0", t)).astype(np.float64) * (t > 1)
    w0 = synth.normal_f32((n,), 0.02, "pin", "w0", t).astype(np.float64)
    m, v, w = oracle.adam_update_f64(g, m0, v0, w0, t=t, **HP)
    rm, rv, rw = _torch_adam(g, m0, v0, w0, t, **HP)
    np.testing.assert_allclose(m, rm, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(v, rv, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(w, rw, rtol=1e-13, atol=1e-300)


def test_adam_step1_closed_form():
    g = np.array([1e-3, -2e-3, 0.0, 5e-9, -1.0])
    w0 = np.array([0.5, 0.5, 0.5, 0.5, 0.5])
    z = np.zeros_like(g)
    m, v, w = oracle.adam_update_f64(g, z, z, w0, t=1, **HP)
    expect = w0 - HP["lr"] * g / (np.abs(g) + HP["eps"])
    np.testing.assert_allclose(w, expect, rtol=1e-15)
    assert w[2] == 0.5  # zero gradient leaves the weight unchanged at step 1
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v, 0.05 * g * g, rtol=1e-15)


def test_adam_step_composition_with_independent_pieces():
    """Full stored-state step == torch Adam on decoded values + brute-force
    scale + torch float8 / numpy float16 requantisation."""
    n = 4099
    gf = synth.normal_f32((n,), 1e-3, "pin", "comp", "g")
    mu = 2.0 ** 10
    _, sg = oracle.compute_scale(oracle.amax(gf), oracle.E5M2, 0, mu=mu)
    gq = oracle.cast(gf, oracle.E5M2, sg)
    w_init = synth.normal_f32((n,), 0.02, "pin", "comp", "w")
    _, s_w = oracle.compute_scale(oracle.amax(w_init), oracle.F16, 0)
    wh = oracle.cast(w_init, oracle.F16, s_w)
    # a non-trivial previous state
    m_prev = synth.normal_f32((n,), 1e-4, "pin", "comp", "m")
    _, s_m = oracle.compute_scale(oracle.amax(m_prev), oracle.E4M3, 0)
    mq = oracle.cast(m_prev, oracle.E4M3, s_m)
    v_prev = np.abs(synth.normal_f32((n,), 1e-7, "pin", "comp", "v"))
    _, s_v = oracle.compute_scale(oracle.amax(v_prev), oracle.F16, 0)
    vh = oracle.cast(v_prev, oracle.F16, s_v)
    t = 3
    out = oracle.adam_step(gq, 1 / sg, mq, s_m, vh, s_v, wh, s_w, t=t, margin=0, **HP)
    assert out["rc"] == 0
    # independent route
    g = _torch_dec(gq, 1) / sg
    m0 = _torch_dec(mq, 0) / s_m
    v0 = vh.view(np.float16).astype(np.float64) / s_v
    w0 = wh.view(np.float16).astype(np.float64) / s_w
    rm, rv, rw = _torch_adam(g, m0, v0, w0, t, **HP)
    for arr, fmt, key in ((rm, oracle.E4M3, "s_m"), (rv, oracle.F16, "s_v"), (rw, oracle.F16, "s_w")):
        a = float(np.max(np.abs(arr)))
        mx = {oracle.E4M3: 448.0, oracle.F16: 65504.0}[fmt]
        assert out[key] == 2.0 ** _brute_exponent(a, mx)
    ref_m = torch.from_numpy(rm * out["s_m"]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref_v = (rv * out["s_v"]).astype(np.float16).view(np.uint16)
    ref_w = (rw * out["s_w"]).astype(np.float16).view(np.uint16)
    # With quantised inputs the exact new value often sits exactly on a rounding
    # midpoint (e.g. 0.9*(-20) + 0.1*640 = 46, halfway between E4M3 44 and 48);
    # two float64 evaluation orders may then land on opposite sides.  Every
    # disagreement must be such a tie and at most one code apart.
    _check_ties(out["mq"], ref_m, rm * out["s_m"], lambda c: oracle.decode_table(0)[c])
    f16 = lambda c: c.view(np.float16).astype(np.float64)
    _check_ties(out["vh"], ref_v, rv * out["s_v"], f16)
    _check_ties(out["wh"], ref_w, rw * out["s_w"], f16)


def _check_ties(ours, ref, exact, dec):
    bad = np.nonzero(ours != ref)[0]
    assert bad.size <= ours.size // 20
    for i in bad:
        a, b = float(dec(ours[i:i + 1])[0]), float(dec(ref[i:i + 1])[0])
        mid = (a + b) / 2
        assert abs(int(ours[i]) - int(ref[i])) == 1
        assert abs(exact[i] - mid) <= 1e-12 * abs(mid), (i, exact[i], a, b)


def test_adam_master_e4m3_copy_matches_independent_route():
    """E4M3 copy of the stored master == torch float8 of (numpy-decoded half /
    s_w * s_q) with s_q from the brute-force exponent of the decoded amax."""
    w = synth.normal_f32((3001,), 0.02, "pin", "wq")
    _, s_w = oracle.compute_scale(oracle.amax(w), oracle.F16, 0)
    wh = oracle.cast(w, oracle.F16, s_w)
    for margin in (0, 2):
        q, s_q = oracle.adam_master_e4m3(wh, s_w, margin)
        dec = wh.view(np.float16).astype(np.float64) / s_w
        e = _brute_exponent(float(np.max(np.abs(dec))), 448.0) - margin
        assert s_q == 2.0 ** e
        ref = torch.from_numpy(dec * s_q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, ref)


def test_adam_sharded_equals_whole_tensor_step():
    """[FP8-LM] 提案手法 O3 (ZeRO-partitioned optimizer state): splitting a
    tensor into slices, taking the max of the slices' amaxes and requantising
    every slice with the scales of that max leaves exactly the state of the
    whole-tensor step.  Outliers in the first and the last slice make the
    slices' own scales differ from the tensor's."""
    n = 4099
    gf = synth.normal_f32((n,), 1e-3, "pin", "shard", "g")
    gf[5] = 0.03      # m and v amax in the first slice
    w_init = synth.normal_f32((n,), 0.02, "pin", "shard", "w")
    w_init[n - 3] = 0.9   # master amax in the last slice
    _, sg = oracle.compute_scale(oracle.amax(gf), oracle.E5M2, 0, mu=2.0 ** 10)
    gq = oracle.cast(gf, oracle.E5M2, sg)
    _, s_w = oracle.compute_scale(oracle.amax(w_init), oracle.F16, 0)
    wh = oracle.cast(w_init, oracle.F16, s_w)
    m_prev = synth.normal_f32((n,), 1e-4, "pin", "shard", "m")
    _, s_m = oracle.compute_scale(oracle.amax(m_prev), oracle.E4M3, 0)
    mq = oracle.cast(m_prev, oracle.E4M3, s_m)
    v_prev = np.abs(synth.normal_f32((n,), 1e-7, "pin", "shard", "v"))
    _, s_v = oracle.compute_scale(oracle.amax(v_prev), oracle.F16, 0)
    vh = oracle.cast(v_prev, oracle.F16, s_v)
    state = (gq, 1 / sg, mq, s_m, vh, s_v, wh, s_w)
    whole = oracle.adam_step(*state, t=2, margin=0, **HP)
    splits = [[(0, 2048), (2048, n)], [(0, 1024), (1024, 3072), (3072, n), (n, n)],
              [(i * 512, min(n, (i + 1) * 512)) for i in range(9)]]
    for bounds in splits:
        own = [oracle.adam_step(gq[lo:hi], 1 / sg, mq[lo:hi], s_m, vh[lo:hi], s_v, wh[lo:hi], s_w,
                                t=2, margin=0, **HP) for lo, hi in bounds if hi > lo]
        assert len({(o["s_m"], o["s_v"], o["s_w"]) for o in own}) > 1  # slices alone disagree
        shard = oracle.adam_step_sharded(*state, t=2, margin=0, bounds=bounds, **HP)
        for k in ("s_m", "s_v", "s_w", "rc"):
            assert shard[k] == whole[k], k
        for k in ("mq", "vh", "wh"):
            assert np.array_equal(shard[k], whole[k]), k
        assert shard["amax"] == whole["amax"]


def test_adam_state_bytes_per_param():
    """[FP8-LM] O2: FP8 grad 1 B + FP8 m1 1 B + FP16 m2 2 B + FP16 master 2 B = 6 B/param."""
    n = 1000
    per = (np.zeros(n, np.uint8).nbytes + np.zeros(n, np.uint8).nbytes
           + np.zeros(n, np.uint16).nbytes + np.zeros(n, np.uint16).nbytes) / n
    assert per == 6.0
    assert 16 / per == pytest.approx(2.67, abs=0.01)


# ---------------------------------------------------------------- scaling variants and the FP8 all-reduce
MIN_SUB = {oracle.E4M3: 2.0 ** -9, oracle.E5M2: 2.0 ** -16, oracle.F16: 2.0 ** -24}  # [OFP8], IEEE binary16
MAXV = {oracle.E4M3: 448.0, oracle.E5M2: 57344.0, oracle.F16: 65504.0}


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2, oracle.F16])
def test_cast_counts_closed_forms(fmt):
    """Underflow: a non-zero value whose code is zero; overflow: |x s| above
    the format's largest finite value.  Hand-placed values with scale 1."""
    t, mx = MIN_SUB[fmt], MAXV[fmt]
    x = np.array([0.0, -0.0, t / 2, -t / 2, t / 4, t * 0.5000001, t, mx, -mx, mx * (1 + 2 ** -20), -2 * mx,
                  np.inf, -np.inf, np.nan, 1.0], dtype=np.float32)
    q, (under, over) = oracle.cast_counts(x, fmt, 1.0)
    x = x.astype(np.float64)
    # t/2 and -t/2 are ties that round to the even code 0; t/4 rounds to 0
    assert under == 3
    # just above max, 2 max, +-inf
    assert over == 4
    # the same elements by an independent route: torch / numpy casts
    if fmt == oracle.F16:
        with np.errstate(over="ignore"):
            ref = x.astype(np.float16).astype(np.float64)
    else:
        ref = torch.from_numpy(np.clip(x, -mx, mx)).to(TORCH_FP8[fmt]).double().numpy()
    assert under == int(np.sum((x != 0) & ~np.isnan(x) & (ref == 0)))
    assert over == int(np.sum(np.abs(x) > mx))


def test_cast_counts_random_vs_torch():
    x = synth.normal_f32((20000,), 1.0, "pin", "counts")
    x[::7] *= 1e-6
    for fmt in (oracle.E4M3, oracle.E5M2):
        for s in (2.0 ** -8, 1.0, 2.0 ** 9):
            q, (under, over) = oracle.cast_counts(x, fmt, s)
            y = x.astype(np.float64) * s
            ref = torch.from_numpy(np.clip(y, -MAXV[fmt], MAXV[fmt])).to(TORCH_FP8[fmt]).double().numpy()
            assert under == int(np.sum((x != 0) & (ref == 0)))
            assert over == int(np.sum(np.abs(y) > MAXV[fmt]))


def test_grad_scale_closed_forms():
    """S = mu * 2^(floor(log2(fmt_max/amax)) - margin): the exponent by brute
    force, mu applied after it (it does not cancel, unlike the cast scale)."""
    assert oracle.grad_scale(1.0, oracle.E5M2, 0, 1.0) == (0, 2.0 ** 15)
    assert oracle.grad_scale(1.0, oracle.E5M2, 0, 2.0 ** -3) == (0, 2.0 ** 12)
    assert oracle.grad_scale(1.0, oracle.E5M2, 1, 2.0 ** -3) == (0, 2.0 ** 11)
    assert oracle.grad_scale(0.0, oracle.E4M3, 0, 2.0 ** -2) == (0, 2.0 ** -2)
    assert oracle.grad_scale(float("inf"), oracle.E4M3, 0, 1.0)[0] != 0
    assert oracle.grad_scale(1e-38, oracle.E5M2, 0, 2.0 ** 8)[1] == 2.0 ** 126
    r = synth.rng("pin", "gscale")
    for a in np.exp(r.uniform(-40, 40, 200)):
        for fmt in (oracle.E4M3, oracle.E5M2):
            for mu_e in (-5, 0, 3):
                e = _brute_exponent(float(a), MAXV[fmt])
                rc, S = oracle.grad_scale(float(a), fmt, 0, 2.0 ** mu_e)
                assert S == 2.0 ** max(-126, min(126, max(-126, min(126, e)) + mu_e))
                # with mu = 1 the payload of the largest element fits, doubled it would not
                if mu_e == 0 and -126 < e < 126:
                    assert a * S <= MAXV[fmt] < 2 * a * S


def _finite_codes(shape, fmt, *key):
    c = synth.rng(*key).integers(0, 256, size=shape, dtype=np.uint8)
    bad = (c & 0x7F) == 0x7F if fmt == oracle.E4M3 else (c & 0x7C) == 0x7C
    c[bad] &= 0x83  # finite, small
    return c


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("nranks", [1, 2, 3, 8])
def test_sum_codes_vs_torch(fmt, nranks):
    rows = _finite_codes((nranks, 5000), fmt, "pin", "sum", fmt, nranks)
    out, (under, over) = oracle.sum_codes(rows, fmt)
    exact = torch.from_numpy(rows).view(TORCH_FP8[fmt]).double().sum(0).numpy()
    # brute force: nearest finite code by a scan of the whole table, ties to the
    # even code, saturating (torch's own double -> float8 path rounds through
    # float32 first, which double-rounds sums like 45055.9997)
    codes = np.arange(256, dtype=np.uint8)
    table = torch.from_numpy(codes).view(TORCH_FP8[fmt]).double().numpy()
    ok = np.isfinite(table)
    codes, table = codes[ok], table[ok]
    y = np.clip(exact, -MAXV[fmt], MAXV[fmt])
    d = np.abs(table[None, :] - y[:, None])
    best = d.min(1, keepdims=True)
    cand = np.where(d == best, codes[None, :].astype(int), 999)
    even = np.where(cand % 2 == 0, cand, 999).min(1)
    pick = np.where((cand != 999).sum(1) > 1, even, cand.min(1))
    # equal-distance pairs are +0 and -0 only when y == 0: take +0
    pick = np.where(y == 0, 0, pick)
    assert np.array_equal(out, pick.astype(np.uint8))
    assert over == int((np.abs(exact) > MAXV[fmt]).sum())
    assert under == 0
    if nranks == 1:  # one rank: the codes come back, a negative zero as +0 (the sum starts at +0)
        assert np.array_equal(out, np.where(rows[0] == 0x80, 0, rows[0]))


def test_sum_codes_specials():
    E5, E4 = oracle.E5M2, oracle.E4M3
    cases = [  # (fmt, codes of the ranks, expected code, expected overflow)
        (E5, [0x7B, 0x7B], 0x7B, 1),   # max + max saturates
        (E5, [0x7B, 0x00], 0x7B, 0),   # exactly max: no overflow
        (E5, [0x01, 0x81], 0x00, 0),   # +-min subnormal cancel: an exact zero is no underflow
        (E5, [0x7C, 0x3C], 0x7B, 1),   # +inf + 1 -> +inf, saturated
        (E5, [0x7C, 0xFC], 0x7F, 0),   # +inf + -inf -> NaN
        (E5, [0x7E, 0x00], 0x7F, 0),   # NaN
        (E4, [0xFF, 0x38], 0x7F, 0),   # NaN (negative NaN code) -> 0x7F
        (E4, [0x7E, 0x7E, 0xFE], 0x7E, 0),  # 448 + 448 - 448 = 448
        (E4, [0x01] * 3, 0x03, 0),     # 3 x 2^-9: an exact subnormal
        (E5, [0x3D] * 3, 0x44, 0),     # 3 x 1.25 = 3.75, halfway between 3.5 (0x43) and 4 (0x44): even
    ]
    for fmt, codes, want, want_over in cases:
        out, (under, over) = oracle.sum_codes(np.array(codes, dtype=np.uint8).reshape(-1, 1), fmt)
        assert (int(out[0]), over, under) == (want, want_over, 0), (fmt, codes)


def test_mu_update_hand_traced():
    args = dict(theta=1e-3, interval=3, mu_min=2.0 ** -4, mu_max=4.0)
    mu, clean = 1.0, 0
    trace = []
    for over in (0, 0, 0, 2, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0):
        mu, clean = oracle.mu_update(mu, clean, over, 1000, **args)
        trace.append((mu, clean))
    assert trace == [(1.0, 1), (1.0, 2), (2.0, 0),    # three clean steps: doubles
                     (1.0, 0),                          # 2 > 1e-3 * 1000: halves
                     (1.0, 1),                          # 1 is not above the threshold
                     (1.0, 2), (2.0, 0), (2.0, 1), (2.0, 2), (4.0, 0),
                     (4.0, 1), (4.0, 2), (4.0, 0), (4.0, 1)]  # held at mu_max
    mu, clean = 2.0 ** -4, 5
    assert oracle.mu_update(mu, clean, 10 ** 6, 1000, **args) == (2.0 ** -4, 0)  # held at mu_min
    assert oracle.mu_update(1.0, 0, 0, 0, **args) == (1.0, 1)  # empty tensor: no overflow


def test_fp8_allreduce_pre_post_auto_hand_built():
    """[FP8-LM] アブレーション研究: dividing by the rank count after the sum
    (post-scaling, mu = 1) overflows where the ranks agree in sign; dividing
    before the cast (pre-scaling, mu = 1/N) underflows small gradients.
    Four ranks, E5M2, amax 1 on every rank."""
    N = 4
    g = np.zeros((N, 4), dtype=np.float32)
    g[:, 0] = 1.0                 # sum 4 x payload: overflows at mu = 1
    g[:, 1] = 2.0 ** -30          # payload 2^-15 at mu = 1, 2^-17 (a tie to 0) at mu = 1/4
    g[:, 2] = [0.5, -0.5, 0.25, -0.25]   # cancels exactly
    g[:, 3] = [0.75, 0.0, 0.0, 0.0]
    post = oracle.fp8_allreduce(list(g), oracle.E5M2, 0, 1.0)
    pre = oracle.fp8_allreduce(list(g), oracle.E5M2, 0, 1.0 / N)
    assert post["S"] == 2.0 ** 15 and pre["S"] == 2.0 ** 13
    assert post["cast_counts"] == (0, 0) and post["sum_counts"] == (0, 1)
    assert pre["cast_counts"] == (4, 0) and pre["sum_counts"] == (0, 0)
    val = lambda r: _torch_dec(r["codes"], oracle.E5M2) / r["S"]
    np.testing.assert_array_equal(val(post), [1.75, 4 * 2.0 ** -30, 0.0, 0.75])   # element 0 saturated
    np.testing.assert_array_equal(val(pre), [4.0, 0.0, 0.0, 0.75])                # element 1 lost
