"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bars: amax, scales and cast bytes bit-exact; GEMM outputs within
1e-3 * sum_k |a b| (+ half an output ULP for 16-bit outputs); fused output
amax bit-exact against the oracle's amax of the GPU's own output; Adam master
weights and second moment within 1 FP16 ULP, first-moment codes within 1 code,
scales bit-equal.  Each stage is fed the GPU's own upstream values.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from fp8_mixed_precision_tensor_b200 import fp8, synth
from _util import (assert_gemm_close, bf16_dev, boundary_samples, code_rank, f16_ulp, f16_vals, tensor_to_np,
                   to_dev)

pytestmark = pytest.mark.gpu

F32 = dict(dtype=torch.float32, device="cuda")
ODT = {fp8.FP8_DT_F32: oracle.DT_F32, fp8.FP8_DT_BF16: oracle.DT_BF16, fp8.FP8_DT_F16: oracle.DT_F16}
OFMT = {fp8.FP8_E4M3: oracle.E4M3, fp8.FP8_E5M2: oracle.E5M2, fp8.FP8_F16S: oracle.F16}


def scalar():
    return torch.zeros(1, **F32)


def host_input(n, dt, key, specials=False):
    """(host array for the oracle, oracle dtype code, device tensor)."""
    b = synth.lognormal_outliers_bf16(n, *key)
    x = synth.bf16_bits_to_f32(b)
    if specials and n >= 8:
        x = x.copy()
        x[[1, n // 2, n - 1]] = [-0.0, 3.0e38 if dt == fp8.FP8_DT_F32 else 60000.0, -7.5]
    if dt == fp8.FP8_DT_F32:
        return x, oracle.DT_F32, to_dev(x)
    if dt == fp8.FP8_DT_BF16:
        bits = synth.to_bf16_bits(x)
        return bits, oracle.DT_BF16, bf16_dev(bits)
    h = np.clip(x, -60000, 60000).astype(np.float16)
    return h.view(np.uint16), oracle.DT_F16, to_dev(h)


# ---------------------------------------------------------------- amax
@pytest.mark.parametrize("dt", [fp8.FP8_DT_F32, fp8.FP8_DT_BF16, fp8.FP8_DT_F16])
@pytest.mark.parametrize("n", [1, 7, 16, 17, 4096 + 5, (1 << 20) + 3])
def test_amax_bit_exact(dt, n):
    h, odt, d = host_input(n, dt, ("amax", dt, n), specials=True)
    a = scalar()
    fp8.fp8_amax(d, a)
    assert a.item() == oracle.amax(h, odt)


def test_amax_empty_and_specials():
    a = scalar()
    a.fill_(5.0)
    fp8.fp8_amax(torch.empty(0, **F32), a)
    assert a.item() == 0.0
    x = torch.tensor([1.0, -float("inf"), 2.0] * 11, **F32)
    fp8.fp8_amax(x, a)
    assert a.item() == math.inf
    x[5] = float("nan")
    fp8.fp8_amax(x, a)
    assert math.isnan(a.item())
    x = torch.tensor([-0.0, 0.0] * 20, **F32)
    fp8.fp8_amax(x, a)
    assert a.item() == 0.0 and math.copysign(1, a.item()) == 1.0


def test_amax_rejects_unaligned():
    x = torch.zeros(100, **F32)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_amax(x[1:], scalar())
    assert e.value.code == fp8.FP8_ERR_UNALIGNED


# ---------------------------------------------------------------- scale
def test_compute_scale_bit_exact_sweep():
    g = synth.rng("scale", "sweep")
    amaxes = list(np.exp(g.uniform(-87, 87, 300)).astype(np.float32))
    amaxes += [0.0, 448.0, 57344.0, 65504.0, 1.0, 1e-45, 1.17e-38, 3.0e38,
               float(np.nextafter(np.float32(448), np.float32(1e9))), float(np.float32(448 * 0.75))]
    am = torch.tensor(amaxes, **F32)
    for fmt in (fp8.FP8_E4M3, fp8.FP8_E5M2, fp8.FP8_F16S):
        for margin in (0, 1, 3):
            for mu in (1.0, 2.0 ** 10, 2.0 ** -4):
                s, inv = torch.zeros_like(am), torch.zeros_like(am)
                for i in range(am.numel()):
                    fp8.fp8_compute_scale(am[i:i + 1], fmt, margin, mu, s[i:i + 1], inv[i:i + 1])
                s_h, inv_h = s.cpu().numpy(), inv.cpu().numpy()
                for i, a in enumerate(amaxes):
                    rc, ref = oracle.compute_scale(float(np.float32(a)), OFMT[fmt], margin, mu=mu)
                    assert rc == 0
                    assert s_h[i] == ref and inv_h[i] == 1.0 / ref, (fmt, margin, mu, a, s_h[i], ref)
    assert fp8.fp8_get_status() == 0


def test_compute_scale_nonfinite_sets_status():
    fp8.fp8_get_status()
    for bad in (float("inf"), float("nan")):
        a = torch.tensor([bad], **F32)
        s, inv = scalar(), scalar()
        fp8.fp8_compute_scale(a, fp8.FP8_E4M3, 0, 1.0, s, inv)
        assert s.item() == 1.0 and inv.item() == 1.0
        assert fp8.fp8_get_status() & fp8.FP8_STATUS_NONFINITE
    assert fp8.fp8_get_status() == 0


def test_compute_scale_rejects_bad_mu_and_margin():
    a, s, inv = scalar(), scalar(), scalar()
    for mu, margin in ((3.0, 0), (0.0, 0), (-2.0, 0), (2.0 ** 40, 0), (1.0, -1)):
        with pytest.raises(fp8.FP8Error) as e:
            fp8.fp8_compute_scale(a, fp8.FP8_E4M3, margin, mu, s, inv)
        assert e.value.code == fp8.FP8_ERR_INVALID_ARG


# ---------------------------------------------------------------- cast
@pytest.mark.parametrize("dt", [fp8.FP8_DT_F32, fp8.FP8_DT_BF16, fp8.FP8_DT_F16])
@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2, fp8.FP8_F16S])
@pytest.mark.parametrize("margin", [0, 1])
def test_amax_scale_cast_chain_bit_exact(dt, fmt, margin):
    n = (1 << 18) + 13
    h, odt, d = host_input(n, dt, ("cast", dt, fmt), specials=True)
    a, s, inv = scalar(), scalar(), scalar()
    q = torch.empty(n, dtype=torch.int16 if fmt == fp8.FP8_F16S else torch.uint8, device="cuda")
    fp8.fp8_amax(d, a)
    fp8.fp8_compute_scale(a, fmt, margin, 1.0, s, inv)
    fp8.fp8_cast(d, fmt, s, q)
    rc, s_ref = oracle.compute_scale(oracle.amax(h, odt), OFMT[fmt], margin)
    assert s.item() == s_ref
    ref = oracle.cast(h, OFMT[fmt], s_ref, odt)
    got = q.cpu().numpy()
    if fmt == fp8.FP8_F16S:
        got = got.view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
def test_cast_saturation_and_specials(fmt):
    vals = np.array([0.0, -0.0, 1.0, -1.0, 448.0, 464.0, 500.0, 57344.0, 61440.0, 1e6, -1e6, np.inf, -np.inf,
                     np.nan, -np.nan, 1e-9, -1e-9, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -16,
                     2.0 ** -17, 3.0e38] * 3, dtype=np.float32)
    d = to_dev(vals)
    s = torch.ones(1, **F32)
    q = torch.empty(vals.size, dtype=torch.uint8, device="cuda")
    fp8.fp8_cast(d, fmt, s, q)
    got = q.cpu().numpy()
    ref = oracle.cast(vals, OFMT[fmt], 1.0)
    nan = np.isnan(vals)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7F) == 0x7F)  # NaN stays NaN


def test_cast_mu_invariance():
    g = synth.normal_f32(((1 << 16) + 3,), 1e-3, "mu")
    d = to_dev(g)
    a = scalar()
    fp8.fp8_amax(d, a)
    codes = []
    for mu in (1.0, 2.0 ** 10, 2.0 ** -4):
        s, inv = scalar(), scalar()
        q = torch.empty(g.size, dtype=torch.uint8, device="cuda")
        fp8.fp8_compute_scale(a, fp8.FP8_E5M2, 0, mu, s, inv)
        fp8.fp8_cast(d, fp8.FP8_E5M2, s, q)
        codes.append(q.cpu().numpy())
        assert s.item() == oracle.compute_scale(oracle.amax(g), oracle.E5M2, 0, mu=mu)[1]
    assert all(np.array_equal(codes[0], c) for c in codes[1:])


def test_cast_rejects_unaligned_and_bad_enums():
    x = torch.zeros(64, **F32)
    q = torch.zeros(64, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, **F32)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_cast(x[1:], fp8.FP8_E4M3, s, q)
    assert e.value.code == fp8.FP8_ERR_UNALIGNED
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_cast(x, 7, s, q)
    assert e.value.code == fp8.FP8_ERR_INVALID_ARG


# ---------------------------------------------------------------- GEMMs
def quantised_linear(M, N, K, key, x_std=1.0, w_std=0.02, dy_std=1e-4):
    """E4M3 X, W and E5M2 dY codes + scales, made by the GPU cast chain."""
    X, W, dY = synth.linear_inputs_f32(M, N, K, x_std, w_std, dy_std, *key)
    out = {}
    for name, host, fmt in (("x", X, fp8.FP8_E4M3), ("w", W, fp8.FP8_E4M3), ("dy", dY, fp8.FP8_E5M2)):
        d = to_dev(host)
        a, s, inv = scalar(), scalar(), scalar()
        q = torch.empty(host.shape, dtype=torch.uint8, device="cuda")
        fp8.fp8_amax(d, a)
        fp8.fp8_compute_scale(a, fmt, 0, 1.0, s, inv)
        fp8.fp8_cast(d, fmt, s, q)
        out[name] = (q, inv)
    return out


OUT_DT = {fp8.FP8_DT_F32: torch.float32, fp8.FP8_DT_BF16: torch.bfloat16, fp8.FP8_DT_F16: torch.float16}

SHAPES = [(256, 256, 256), (128, 256, 128), (16, 16, 16), (272, 400, 208), (384, 528, 1040),
          (1024, 768, 4096)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("out_dt", [fp8.FP8_DT_F32, fp8.FP8_DT_BF16])
def test_linear_gemms_vs_oracle(shape, out_dt):
    M, N, K = shape
    q = quantised_linear(M, N, K, ("gemm", shape))
    (xq, xi), (wq, wi), (dyq, dyi) = q["x"], q["w"], q["dy"]
    tdt = OUT_DT[out_dt]
    y = torch.empty((M, N), dtype=tdt, device="cuda")
    dx = torch.empty((M, K), dtype=tdt, device="cuda")
    dw = torch.empty((N, K), dtype=tdt, device="cuda")
    ya, dxa, dwa = scalar(), scalar(), scalar()
    fp8.fp8_linear_fwd(xq, xi, wq, wi, y, ya)
    fp8.fp8_linear_dgrad(dyq, dyi, wq, wi, dx, dxa)
    fp8.fp8_linear_wgrad(dyq, dyi, xq, xi, dw, dwa)
    assert fp8.fp8_get_status() == 0
    h = {k: (v[0].cpu().numpy(), float(v[1].item())) for k, v in q.items()}
    refs = {
        "fwd": oracle.linear_fwd(h["x"][0], h["x"][1], h["w"][0], h["w"][1], M, N, K),
        "dgrad": oracle.linear_dgrad(h["dy"][0], h["dy"][1], h["w"][0], h["w"][1], M, N, K),
        "wgrad": oracle.linear_wgrad(h["dy"][0], h["dy"][1], h["x"][0], h["x"][1], M, N, K),
    }
    for name, out, amax in (("fwd", y, ya), ("dgrad", dx, dxa), ("wgrad", dw, dwa)):
        ref, rabs = refs[name]
        got = tensor_to_np(out)
        assert_gemm_close(got, ref, rabs, tdt, f"{name} {shape}")
        # fused amax == amax of the GPU's own stored output, bit-exact
        assert amax.item() == float(np.max(np.abs(got))), name


@pytest.mark.parametrize("shape", [(2320, 2064, 400), (2048, 4096, 512), (2320, 4624, 4112)])
def test_linear_gemms_pair_kernel_sampled(shape):
    """Shapes with enough 256x256 (first two) or 256x512 (last: all three
    GEMMs) tiles to run the two-CTA kernels, ragged edges included; the oracle
    computes sampled outputs one by one."""
    M, N, K = shape
    q = quantised_linear(M, N, K, ("gemm-pair", shape))
    (xq, xi), (wq, wi), (dyq, dyi) = q["x"], q["w"], q["dy"]
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ya, dxa, dwa = scalar(), scalar(), scalar()
    fp8.fp8_linear_fwd(xq, xi, wq, wi, y, ya)
    fp8.fp8_linear_dgrad(dyq, dyi, wq, wi, dx, dxa)
    fp8.fp8_linear_wgrad(dyq, dyi, xq, xi, dw, dwa)
    assert fp8.fp8_get_status() == 0
    h = {k: (v[0].cpu().numpy(), float(v[1].item())) for k, v in q.items()}
    for name, out, amax, (rows, cols), fn in (
            ("fwd", y, ya, (M, N), lambda smp: oracle.linear_fwd(h["x"][0], h["x"][1], h["w"][0], h["w"][1],
                                                                 M, N, K, samples=smp)),
            ("dgrad", dx, dxa, (M, K), lambda smp: oracle.linear_dgrad(h["dy"][0], h["dy"][1], h["w"][0],
                                                                       h["w"][1], M, N, K, samples=smp)),
            ("wgrad", dw, dwa, (N, K), lambda smp: oracle.linear_wgrad(h["dy"][0], h["dy"][1], h["x"][0],
                                                                       h["x"][1], M, N, K, samples=smp))):
        r, c = boundary_samples(rows, cols, 3000, (name, shape), tile_c=(256, 512))
        ref, rabs = fn((r, c))
        got = tensor_to_np(out)
        assert_gemm_close(got[r, c], ref, rabs, out.dtype, f"{name} {shape}")
        assert amax.item() == float(np.max(np.abs(got))), name


def test_linear_wide_kernel_16bit_outputs_and_bias():
    """The 256x512 two-CTA kernel with every 16-bit output path: fwd with a
    bias into fp16, dgrad into fp16, wgrad into bf16 (ragged edges)."""
    M, N, K = 2320, 4624, 528
    q = quantised_linear(M, N, K, ("gemm-wide16",))
    (xq, xi), (wq, wi), (dyq, dyi) = q["x"], q["w"], q["dy"]
    bias = synth.normal_f32((N,), 0.5, "wide16", "b")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.float16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    ya, dxa, dwa = scalar(), scalar(), scalar()
    fp8.fp8_linear_fwd(xq, xi, wq, wi, y, ya, bias=to_dev(bias))
    fp8.fp8_linear_dgrad(dyq, dyi, wq, wi, dx, dxa)
    fp8.fp8_linear_wgrad(dyq, dyi, xq, xi, dw, dwa)
    assert fp8.fp8_get_status() == 0
    h = {k: (v[0].cpu().numpy(), float(v[1].item())) for k, v in q.items()}
    for name, out, amax, (rows, cols), fn in (
            ("fwd", y, ya, (M, N), lambda smp: oracle.linear_fwd(h["x"][0], h["x"][1], h["w"][0], h["w"][1],
                                                                 M, N, K, bias=bias.astype(np.float64),
                                                                 samples=smp)),
            ("dgrad", dx, dxa, (M, K), lambda smp: oracle.linear_dgrad(h["dy"][0], h["dy"][1], h["w"][0],
                                                                       h["w"][1], M, N, K, samples=smp)),
            ("wgrad", dw, dwa, (N, K), lambda smp: oracle.linear_wgrad(h["dy"][0], h["dy"][1], h["x"][0],
                                                                       h["x"][1], M, N, K, samples=smp))):
        r, c = boundary_samples(rows, cols, 3000, (name, "wide16"), tile_c=(256, 512))
        ref, rabs = fn((r, c))
        got = tensor_to_np(out) if out.dtype != torch.float16 else out.double().cpu().numpy()
        assert_gemm_close(got[r, c], ref, rabs, out.dtype, f"{name} wide16")
        assert amax.item() == float(np.max(np.abs(got))), name


def test_linear_fwd_bias_f16_out():
    M, N, K = 256, 272, 128
    q = quantised_linear(M, N, K, ("bias",))
    (xq, xi), (wq, wi) = q["x"], q["w"]
    bias = synth.normal_f32((N,), 0.5, "bias", "b")
    for bdt, tb in ((fp8.FP8_DT_F32, to_dev(bias)), (fp8.FP8_DT_BF16, to_dev(bias).bfloat16())):
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        ya = scalar()
        fp8.fp8_linear_fwd(xq, xi, wq, wi, y, ya, bias=tb)
        b_used = tb.double().cpu().numpy()
        ref, rabs = oracle.linear_fwd(xq.cpu().numpy(), xi.item(), wq.cpu().numpy(), wi.item(), M, N, K,
                                      bias=b_used)
        got = y.double().cpu().numpy()
        assert_gemm_close(got, ref, rabs, torch.float16, f"bias {bdt}")
        assert ya.item() == float(np.max(np.abs(got)))


@pytest.mark.parametrize("shape", [(256, 256, 256), (272, 400, 208), (1024, 768, 4096), (1024, 16384, 2048)])
def test_wgrad_round_to_odd_output_feeds_the_same_gradient_codes(shape):
    """The bfloat16 round-to-odd wgrad output (FP8_DT_BF16_RTO) is, bit for
    bit, the round-to-odd image of the same kernel's float32 output (the
    accumulation does not change with the output type), its fused amax is the
    amax of the stored values, and the E5M2 gradient cast of it -- scale,
    codes and under/overflow counts -- equals the cast of the float32 output.
    The shapes run the one-CTA, pair and wide kernels."""
    M, N, K = shape
    q = quantised_linear(M, N, K, ("rto", M, N, K))
    (dyq, dy_inv), (xq, x_inv) = q["dy"], q["x"]
    dw32, a32 = torch.empty((N, K), **F32), scalar()
    fp8.fp8_linear_wgrad(dyq, dy_inv, xq, x_inv, dw32, a32)
    dwb, ab = torch.empty((N, K), dtype=torch.bfloat16, device="cuda"), scalar()
    fp8.fp8_linear_wgrad(dyq, dy_inv, xq, x_inv, dwb, ab, rto=True)
    u = dw32.cpu().numpy().view(np.uint32)
    want = (u >> 16).astype(np.uint16) | ((u & 0xFFFF) != 0).astype(np.uint16)
    got = dwb.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    stored = (got.astype(np.uint32) << 16).view(np.float32)
    assert ab.item() == float(np.max(np.abs(stored)))
    mu = torch.full((1,), 2.0 ** 10, **F32)
    res = []
    for g, a in ((dw32, a32), (dwb, ab)):
        S, inv, counts = scalar(), scalar(), torch.zeros(2, dtype=torch.int64, device="cuda")
        codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        fp8.fp8_grad_cast(g, fp8.FP8_E5M2, a, 0, mu, S, inv, codes, counts)
        res.append((S.item(), codes.cpu().numpy(), tuple(counts.tolist())))
    assert res[0][0] == res[1][0] and res[0][2] == res[1][2]
    assert np.array_equal(res[0][1], res[1][1])
    with pytest.raises(TypeError):  # a round-to-odd output is bfloat16
        fp8.fp8_linear_wgrad(dyq, dy_inv, xq, x_inv, dw32, a32, rto=True)


def test_gemm_exact_integer_operands():
    """Codes for +-1, +-2 only: every partial sum is an exact integer, so the
    FP32 accumulation must equal the oracle exactly."""
    M, N, K = 256, 256, 2048
    g = synth.rng("gemm", "int")
    pick = np.array([0x38, 0xB8, 0x40, 0xC0], np.uint8)
    xq = pick[g.integers(0, 4, (M, K))]
    wq = pick[g.integers(0, 4, (N, K))]
    one = torch.ones(1, **F32)
    y = torch.empty((M, N), **F32)
    fp8.fp8_linear_fwd(to_dev(xq), one, to_dev(wq), one, y)
    ref, _ = oracle.linear_fwd(xq, 1.0, wq, 1.0, M, N, K)
    assert np.array_equal(y.cpu().numpy().astype(np.float64), ref)


def test_gemm_rejects_unsupported_shapes():
    a = torch.zeros((32, 24), dtype=torch.uint8, device="cuda")
    b = torch.zeros((32, 24), dtype=torch.uint8, device="cuda")
    y = torch.zeros((32, 32), **F32)
    one = torch.ones(1, **F32)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_linear_fwd(a, one, b, one, y)
    assert e.value.code == fp8.FP8_ERR_UNSUPPORTED


def test_gemm_empty_rows_writes_zero_amax():
    a = torch.zeros((0, 32), dtype=torch.uint8, device="cuda")
    b = torch.zeros((32, 32), dtype=torch.uint8, device="cuda")
    y = torch.zeros((0, 32), **F32)
    ya = torch.full((1,), 3.0, **F32)
    one = torch.ones(1, **F32)
    fp8.fp8_linear_fwd(a, one, b, one, y, ya)
    assert ya.item() == 0.0


# ---------------------------------------------------------------- Adam
HP = dict(lr=1e-4, beta1=0.9, beta2=0.95, eps=1e-8)


def make_adam_state(sizes, key, steps_done=0, g_host=None):
    """Per chunk: E5M2 grads (mu = 2^10) and a stored state built by the GPU
    cast chain from seeded fp32 tensors (zero moments when steps_done == 0).
    The fp32 gradients are ~N(0, 1e-3), or g_host[ci] when given."""
    chunks, host = [], []
    for ci, n in enumerate(sizes):
        gf = synth.adam_grad_f32(n, 1e-3, *key, ci, "g") if g_host is None else g_host[ci]
        wf = synth.normal_f32((n,), 0.02, *key, ci, "w")
        st = {}
        for name, arr, fmt, mu in (("g", gf, fp8.FP8_E5M2, 2.0 ** 10), ("w", wf, fp8.FP8_F16S, 1.0)):
            d = to_dev(arr)
            a, s, inv = scalar(), scalar(), scalar()
            q = torch.empty(n, dtype=torch.uint8 if fmt != fp8.FP8_F16S else torch.int16, device="cuda")
            fp8.fp8_amax(d, a)
            fp8.fp8_compute_scale(a, fmt, 0, mu, s, inv)
            fp8.fp8_cast(d, fmt, s, q)
            st[name] = (q, s, inv)
        if steps_done:
            mf = synth.normal_f32((n,), 1e-4, *key, ci, "m")
            vf = np.abs(synth.normal_f32((n,), 1e-7, *key, ci, "v"))
            for name, arr, fmt in (("m", mf, fp8.FP8_E4M3), ("v", vf, fp8.FP8_F16S)):
                d = to_dev(arr)
                a, s, inv = scalar(), scalar(), scalar()
                q = torch.empty(n, dtype=torch.uint8 if fmt != fp8.FP8_F16S else torch.int16, device="cuda")
                fp8.fp8_amax(d, a)
                fp8.fp8_compute_scale(a, fmt, 0, 1.0, s, inv)
                fp8.fp8_cast(d, fmt, s, q)
                st[name] = (q, s)
        else:
            st["m"] = (torch.zeros(n, dtype=torch.uint8, device="cuda"), torch.ones(1, **F32))
            st["v"] = (torch.zeros(n, dtype=torch.int16, device="cuda"), torch.ones(1, **F32))
        c = fp8.AdamChunk(st["g"][0], st["g"][2], st["m"][0], st["m"][1], st["v"][0], st["v"][1],
                          st["w"][0], st["w"][1])
        chunks.append(c)
    return chunks


def snapshot(c):
    return dict(g=c.g.cpu().numpy(), g_inv=c.g_inv.item(), m=c.m.cpu().numpy(), s_m=c.m_scale.item(),
                v=c.v.cpu().numpy().view(np.uint16), s_v=c.v_scale.item(),
                w=c.w.cpu().numpy().view(np.uint16), s_w=c.w_scale.item())


# The kernel evaluates the update in binary32 with every operation rounded to
# nearest; counting those roundings (and the binary32 representation of lr,
# beta1, beta2, eps and the bias corrections) bounds its step's error by
# STEP_ROUNDINGS * 2^-24 * dw_abs, where dw_abs is the step computed from the
# magnitudes of m's two terms, lr (b1 |m0| + (1 - b1) |g|) / (1 - b1^t) /
# (sqrt(v_hat) + eps).  The master is compared at 1 FP16 ULP plus that term
# (which only matters where the step cancels most of the weight).
STEP_ROUNDINGS = 24
MAX_TIES = 1  # scale ties tolerated per test (each is still checked element by element)
FMAX_ADAM = (("s_m", 448.0), ("s_v", 65504.0), ("s_w", 65504.0))


def adam_step_magnitude(before, step, hp=HP):
    """dw_abs of every element, float64, from the decoded stored state."""
    g = oracle.decode_table(oracle.E5M2)[before["g"]] * before["g_inv"]
    m0 = oracle.decode_table(oracle.E4M3)[before["m"]] / before["s_m"]
    v0 = f16_vals(before["v"]) / before["s_v"]
    b1, b2 = hp["beta1"], hp["beta2"]
    v = b2 * v0 + (1 - b2) * g * g
    den = np.sqrt(v / (1 - b2 ** step)) + hp["eps"]
    return hp["lr"] * (b1 * np.abs(m0) + (1 - b1) * np.abs(g)) / (1 - b1 ** step) / den


def _slice(state, lo, hi):
    return {k: (v[lo:hi] if isinstance(v, np.ndarray) else v) for k, v in state.items()}


def check_adam_chunk(before, c, step, margin=0, ties=None, slices=1, hp=HP):
    """Oracle step from `before` against the chunk's state now.  Scales must be
    bit-equal; a mismatch is allowed only where the oracle's float64 amax lies
    within 4 binary32 ULPs of a scale threshold (a tie).  A tie is appended to
    `ties` (a failure when `ties` is None) and the elements are still compared,
    against the oracle re-run at the GPU's scale for the tied tensor.
    slices > 1 bounds the oracle's memory for large chunks: the tensor's new
    amaxes are the maximum of its slices' (the element-sharded oracle step),
    then every slice is requantised with them and compared on its own."""
    after = snapshot(c)
    n = before["g"].size
    bounds = [(n * k // slices, n * (k + 1) // slices) for k in range(slices)]

    def run(b, amax_in=None):
        return oracle.adam_step(b["g"], b["g_inv"], b["m"], b["s_m"], b["v"], b["s_v"], b["w"], b["s_w"],
                                t=step, margin=margin, amax_in=amax_in, **hp)

    first = run(before) if slices == 1 else None
    amax = first["amax"] if slices == 1 else tuple(
        max(x) if not any(np.isnan(x)) else float("nan")
        for x in zip(*(run(_slice(before, lo, hi))["amax"] for lo, hi in bounds)))
    ref_scales = first if slices == 1 else run(_slice(before, 0, bounds[0][1] if n else 0), amax_in=amax)
    tied = []
    for j, (key, fmax) in enumerate(FMAX_ADAM):
        if after[key] != ref_scales[key]:
            e = oracle.floor_log2_ratio(amax[j], fmax)
            thresh = fmax * 2.0 ** (-e)
            assert abs(amax[j] - thresh) <= 4 * np.spacing(np.float32(thresh)), (key, after[key], ref_scales[key])
            tied.append(j)
    amax_in = None if slices == 1 else amax
    if tied:
        assert ties is not None, f"scale tie at an oracle amax on a threshold: {tied}"
        ties.append((step, tied))
        amax_in = list(amax)
        for j in tied:
            amax_in[j] = FMAX_ADAM[j][1] / (after[FMAX_ADAM[j][0]] * 2.0 ** margin)
        amax_in = tuple(amax_in)
    for lo, hi in bounds:
        b, a = _slice(before, lo, hi), _slice(after, lo, hi)
        out = first if (slices == 1 and amax_in is None) else run(b, amax_in)
        assert (a["s_m"], a["s_v"], a["s_w"]) == (out["s_m"], out["s_v"], out["s_w"])
        # master within 1 FP16 ULP (+ the binary32 step term); second moment within 1 FP16 ULP
        slack = STEP_ROUNDINGS * 2.0 ** -24 * adam_step_magnitude(b, step, hp)
        for key, okey, skey in (("w", "wh", "s_w"), ("v", "vh", "s_v")):
            ref = f16_vals(out[okey]) / out[skey]
            got = f16_vals(a[key]) / a[skey]
            ulp = f16_ulp(f16_vals(out[okey])) / out[skey]
            if key == "w":
                ulp = ulp * (1.0 + 2.0 ** -12) + slack
            bad = np.abs(got - ref) > ulp
            assert not np.any(bad), (key, lo, np.count_nonzero(bad), got[bad][:4], ref[bad][:4])
        # first moment within 1 code (scales equal)
        assert np.all(np.abs(code_rank(a["m"]) - code_rank(out["mq"])) <= 1), lo
    return first if slices == 1 and amax_in is None else out


@pytest.mark.parametrize("sizes", [[65536], [1, 7, 16, 4099, 65536 + 5, 0], [300000, 4096 * 3]])
@pytest.mark.parametrize("steps_done", [0, 4])
def test_adam_step_vs_oracle(sizes, steps_done):
    chunks = make_adam_state(sizes, ("adam", len(sizes), steps_done), steps_done)
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(chunks)) // 4, **F32)
    step = steps_done + 1
    before = [snapshot(c) for c in chunks]
    fp8.fp8_adam_step(chunks, step=step, margin=0, workspace=ws, **HP)
    assert fp8.fp8_get_status() == 0
    ties = []
    for b, c in zip(before, chunks):
        if b["g"].size:
            check_adam_chunk(b, c, step, ties=ties)
    assert len(ties) <= MAX_TIES, ties


def test_adam_subnormal_second_moment():
    """Gradients of magnitude in [2^-66, 2^-65): the new second moment
    (1 - beta2) g^2 lies in [2^-136.3, 2^-134.3), a binary32 subnormal, and
    its scale is the clamped 2^126.  The codes and scales match the oracle, so
    the packed multiply-adds keep subnormals (flushed, v would be 0 with scale
    1), and so does the correctly rounded square root; the step matches
    (sqrt(v_hat) ~ 2^-66 is far below half an ULP of eps = 1e-8).  The stored
    v * 2^126 lies in [2^-10.3, 2^-8.3), where binary32's subnormal spacing
    (2^-149, i.e. 2^-23 after scaling) is far below an FP16 ULP."""
    n = 65536 + 3
    g = synth.rng("adam-subnormal", "g")
    gf = (np.where(g.random(n) < 0.5, -1.0, 1.0) * 2.0 ** -66 * (1.0 + g.random(n))).astype(np.float32)
    chunks = make_adam_state([n], ("adam-subnormal",), g_host=[gf])
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(1) // 4, **F32)
    before = snapshot(chunks[0])
    fp8.fp8_adam_step(chunks, step=1, margin=0, workspace=ws, **HP)
    assert fp8.fp8_get_status() == 0
    out = check_adam_chunk(before, chunks[0], 1)
    assert 0.0 < out["amax"][1] < 2.0 ** -126  # the oracle's new amax(v) is subnormal
    assert snapshot(chunks[0])["s_v"] == 2.0 ** 126  # its scale, clamped


def test_adam_three_steps_stage_parity():
    """Each step's oracle input is the GPU's own stored state from the step before."""
    chunks = make_adam_state([50000, 12345], ("adam3",))
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(2) // 4, **F32)
    for step in (1, 2, 3):
        before = [snapshot(c) for c in chunks]
        fp8.fp8_adam_step(chunks, step=step, margin=1, workspace=ws, **HP)
        for b, c in zip(before, chunks):
            out = oracle.adam_step(b["g"], b["g_inv"], b["m"], b["s_m"], b["v"], b["s_v"], b["w"], b["s_w"],
                                   t=step, margin=1, **HP)
            a = snapshot(c)
            assert (a["s_m"], a["s_v"], a["s_w"]) == (out["s_m"], out["s_v"], out["s_w"])


def test_adam_many_chunks_multiple_launches():
    sizes = [37 + 16 * i for i in range(300)]  # > 224 chunks: two launch groups
    chunks = make_adam_state(sizes, ("adam-many",))
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(chunks)) // 4, **F32)
    before = [snapshot(c) for c in chunks]
    fp8.fp8_adam_step(chunks, step=1, margin=0, workspace=ws, **HP)
    ties = []
    for i in (0, 1, 255, 256, 299):
        check_adam_chunk(before[i], chunks[i], 1, ties=ties)
    assert len(ties) <= MAX_TIES, ties


def test_adam_rejects_bad_args():
    chunks = make_adam_state([64], ("adam-bad",))
    ws = torch.zeros(16, **F32)
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_adam_step(chunks, step=0, margin=0, workspace=ws, **HP)
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_adam_step(chunks, step=1, margin=0, workspace=ws[:3], **HP)


# ---------------------------------------------------------------- Adam: tracked master amax, E4M3 copy
def _with_tracking(chunks, wq=False, track=True):
    out = []
    for c in chunks:
        n = c.g.numel()
        extra = dict(w_amax=torch.full((1,), -1.0, **F32)) if track else {}
        if wq:
            extra.update(wq=torch.empty(n, dtype=torch.uint8, device="cuda"), wq_scale=scalar(), wq_inv=scalar())
        out.append(fp8.AdamChunk(c.g, c.g_inv, c.m, c.m_scale, c.v, c.v_scale, c.w, c.w_scale, **extra))
    return out


def _stored_amax(snap):
    return float(np.max(np.abs(f16_vals(snap["w"])))) / snap["s_w"]


@pytest.mark.parametrize("sizes", [[65536, 4099], [300000, 7, 16]])
def test_adam_tracked_master_amax_matches_untracked(sizes):
    """Step 1 with the tracked amax unknown (full path), steps 2-3 with it known
    (the first pass skips the master): every step leaves exactly the state of
    the untracked step, and the tracked value is the amax of the stored master."""
    ref = make_adam_state(sizes, ("adam-track",))
    trk = _with_tracking(make_adam_state(sizes, ("adam-track",)), wq=True)
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(ref)) // 4, **F32)
    ties = []
    for step in (1, 2, 3):
        before = [snapshot(c) for c in trk]
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        fp8.fp8_adam_step(trk, step=step, margin=0, workspace=ws, **HP)
        assert fp8.fp8_get_status() == 0
        for b, r, t in zip(before, ref, trk):
            sr, st = snapshot(r), snapshot(t)
            for k in ("m", "v", "w", "s_m", "s_v", "s_w"):
                assert np.array_equal(np.asarray(sr[k]), np.asarray(st[k])), (step, k)
            assert t.w_amax.item() == _stored_amax(st)
            q, s_q = oracle.adam_master_e4m3(st["w"], st["s_w"], 0)
            assert t.wq_scale.item() == s_q and t.wq_inv.item() == 1.0 / s_q
            assert np.array_equal(t.wq.cpu().numpy(), q)
            if b["g"].size:
                check_adam_chunk(b, t, step, ties=ties)
    assert len(ties) <= MAX_TIES, ties


def test_adam_mixed_tracked_and_untracked_chunks_in_one_launch():
    """Only some chunks track their master amax: the others take the plain
    path in the same launches, and no consistency check misfires."""
    sizes = [65536, 4099, 300000]
    ref = make_adam_state(sizes, ("adam-mixed",))
    mix = make_adam_state(sizes, ("adam-mixed",))
    trk = _with_tracking(mix[1:2], wq=True)
    mix = [mix[0], trk[0], mix[2]]
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(3) // 4, **F32)
    for step in (1, 2, 3):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        fp8.fp8_adam_step(mix, step=step, margin=0, workspace=ws, **HP)
        assert fp8.fp8_get_status() == 0
        for r, m in zip(ref, mix):
            sr, sm = snapshot(r), snapshot(m)
            for k in ("m", "v", "w", "s_m", "s_v", "s_w"):
                assert np.array_equal(np.asarray(sr[k]), np.asarray(sm[k])), (step, k)
        assert mix[1].w_amax.item() == _stored_amax(snapshot(mix[1]))


def test_adam_tracked_amax_straddling_a_threshold_takes_the_exact_pass():
    """Master amax just below an FP16 scale threshold with steps large enough
    to cross it: the bounds cannot fix the exponent, so the master is re-read;
    the result must still equal the oracle's."""
    n = 8192
    thresh = 65504.0 * 2.0 ** -17  # new scale 2^17 below it, 2^16 above
    w = synth.normal_f32((n,), 0.1, "straddle", "w")
    w[17] = np.float32(thresh * (1 - 2e-4))
    chunks = make_adam_state([n], ("straddle",))
    c = chunks[0]
    d = to_dev(w)
    a, s, inv = scalar(), scalar(), scalar()
    fp8.fp8_amax(d, a)
    fp8.fp8_compute_scale(a, fp8.FP8_F16S, 0, 1.0, c.w_scale, inv)
    fp8.fp8_cast(d, fp8.FP8_F16S, c.w_scale, c.w)
    trk = _with_tracking(chunks)
    trk[0].w_amax.fill_(_stored_amax(snapshot(trk[0])))
    before = snapshot(trk[0])
    hp = dict(HP, lr=1e-1)  # step |dw| ~ 0.1 >> distance to the threshold
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(1) // 4, **F32)
    fp8.fp8_adam_step(trk, step=1, margin=0, workspace=ws, **hp)
    assert fp8.fp8_get_status() == 0
    out = oracle.adam_step(before["g"], before["g_inv"], before["m"], before["s_m"], before["v"], before["s_v"],
                           before["w"], before["s_w"], t=1, margin=0, **hp)
    after = snapshot(trk[0])
    assert (after["s_m"], after["s_v"], after["s_w"]) == (out["s_m"], out["s_v"], out["s_w"])
    ref = f16_vals(out["wh"]) / out["s_w"]
    got = f16_vals(after["w"]) / after["s_w"]
    assert np.all(np.abs(got - ref) <= f16_ulp(f16_vals(out["wh"])) / out["s_w"])
    assert trk[0].w_amax.item() == _stored_amax(after)


def _set_master(c, w):
    """Store host weights w as the chunk's FP16 master (scale from their amax)."""
    d = to_dev(w)
    a, inv = scalar(), scalar()
    fp8.fp8_amax(d, a)
    fp8.fp8_compute_scale(a, fp8.FP8_F16S, 0, 1.0, c.w_scale, inv)
    fp8.fp8_cast(d, fp8.FP8_F16S, c.w_scale, c.w)


@pytest.mark.parametrize("wq", [False, True])
def test_adam_estimated_stats_equal_exact_stats(wq):
    """The whole step decides each untracked chunk's master scale from an
    estimated amax and its error interval; the phased step (stats, then
    apply) computes the exact amax.  Both must leave the same state bit for
    bit: for a chunk whose largest weight sits exactly on an FP16 scale
    threshold and does not move (zero gradient and moment), one whose largest
    weight steps from above the threshold onto it (within a few binary32
    ULPs: the interval cannot decide either, so the exact pass runs), one
    whose largest weight sits on a threshold of the E4M3 copy's scale (448 *
    2^-10: only the copy's interval is ambiguous), and a plain chunk."""
    n = 8192
    thresh = 65504.0 * 2.0 ** -17  # 0.499755859375: scale 2^17 at or below it, 2^16 above
    sets = []
    for _ in range(2):
        chunks = make_adam_state([n] * 4, ("estimate",))
        for k, c in enumerate(chunks):
            w = synth.normal_f32((n,), 0.05, "estimate", k, "w")
            if k < 3:
                # 0.5: the next FP16 value above the threshold at scale 2^16
                w[100 + k] = (thresh, 0.5, 448.0 * 2.0 ** -10)[k]
            _set_master(c, w)
        chunks[0].g[100] = 0      # does not move
        chunks[1].g[101] = 0x3C   # E5M2 1.0: a positive gradient, the step goes down
        chunks[2].g[102] = 0      # does not move
        if wq:
            chunks = _with_tracking(chunks, wq=True, track=False)
        sets.append(chunks)
    whole, phased = sets
    # step 1 from zero moments: dw = -lr g / (|g| + eps); this lr makes the
    # second chunk's 0.5 land on the threshold (0.5 - 2^-12) up to roundings
    g = float(whole[1].g_inv.item())
    hp = dict(HP, lr=2.0 ** -12 * (g + HP["eps"]) / g)
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(4) // 4, **F32)
    ws2 = torch.zeros_like(ws)
    ties = []
    for step in (1, 2):
        before = [snapshot(c) for c in whole]
        fp8.fp8_adam_step(whole, step=step, margin=0, workspace=ws, **hp)
        fp8.fp8_adam_stats(phased, step=step, margin=0, workspace=ws2, **hp)
        fp8.fp8_adam_apply(phased, step=step, margin=0, workspace=ws2, **hp)
        assert fp8.fp8_get_status() == 0
        for b, x, y in zip(before, whole, phased):
            sx, sy = snapshot(x), snapshot(y)
            for k in ("m", "v", "w", "s_m", "s_v", "s_w"):
                assert np.array_equal(np.asarray(sx[k]), np.asarray(sy[k])), (step, k)
            if wq:
                assert x.wq_scale.item() == y.wq_scale.item()
                assert np.array_equal(x.wq.cpu().numpy(), y.wq.cpu().numpy())
        if step == 1:
            # both threshold chunks really ended at the threshold
            for c in whole[:2]:
                assert abs(_stored_amax(snapshot(c)) - thresh) <= thresh * 2.0 ** -10
            assert _stored_amax(snapshot(whole[2])) == 448.0 * 2.0 ** -10
        # the oracle agrees (the threshold chunks may tie in float64)
        for b, x in zip(before, whole):
            check_adam_chunk(b, x, step, ties=ties, hp=hp)
    assert len(ties) <= 2 + MAX_TIES, ties


@pytest.mark.parametrize("dt", [fp8.FP8_DT_F32, fp8.FP8_DT_BF16])
@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2, fp8.FP8_F16S])
@pytest.mark.parametrize("mu,margin", [(1.0, 0), (2.0 ** 10, 1), (2.0 ** -4, 0)])
def test_fused_scale_cast_equals_scale_then_cast(dt, fmt, mu, margin):
    n = (1 << 17) + 9
    h, odt, d = host_input(n, dt, ("fused", dt, fmt), specials=True)
    a = scalar()
    fp8.fp8_amax(d, a)
    qt = torch.int16 if fmt == fp8.FP8_F16S else torch.uint8
    s1, i1, s2, i2 = scalar(), scalar(), scalar(), scalar()
    q1, q2 = torch.empty(n, dtype=qt, device="cuda"), torch.empty(n, dtype=qt, device="cuda")
    fp8.fp8_compute_scale(a, fmt, margin, mu, s1, i1)
    fp8.fp8_cast(d, fmt, s1, q1)
    fp8.fp8_scale_cast(d, fmt, a, margin, mu, s2, i2, q2)
    assert (s1.item(), i1.item()) == (s2.item(), i2.item())
    assert torch.equal(q1, q2)
    rc, s_ref = oracle.compute_scale(oracle.amax(h, odt), OFMT[fmt], margin, mu=mu)
    assert s2.item() == s_ref
    ref = oracle.cast(h, OFMT[fmt], s_ref, odt)
    got = q2.cpu().numpy()
    assert np.array_equal(got.view(np.uint16) if fmt == fp8.FP8_F16S else got, ref)
    # n == 0 still publishes the scales
    s3, i3 = scalar(), scalar()
    fp8.fp8_scale_cast(torch.empty(0, **F32), fmt, a, margin, mu, s3, i3, torch.empty(0, dtype=qt, device="cuda"))
    assert s3.item() == s2.item()


# ---------------------------------------------------------------- Adam: element-sharded step
def _reduce_max_int32(workspaces):
    """Stand-in for the MAX all-reduce over ranks: every rank's workspace gets
    the element-wise max of all of them, compared as int32 words."""
    red = torch.stack([w.view(torch.int32) for w in workspaces]).amax(0)
    for w in workspaces:
        w.view(torch.int32).copy_(red)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("wq", [False, True])
def test_adam_sharded_ranks_equal_whole_tensor_step(world, wq):
    """"FP8-LM", 提案手法 O3: ranks holding slices of every tensor, run one
    after another on this GPU (stats on each, a max over their workspaces,
    apply on each), end with exactly the state and scales of the
    whole-tensor step, over two steps."""
    from fp8_mixed_precision_tensor_b200 import zero

    sizes = [65536 + 5, 4099, 16, 300000]
    ref = make_adam_state(sizes, ("adam-shard",))
    full = make_adam_state(sizes, ("adam-shard",))
    if wq:
        ref = [fp8.AdamChunk(c.g, c.g_inv, c.m, c.m_scale, c.v, c.v_scale, c.w, c.w_scale, None,
                             torch.empty(c.g.numel(), dtype=torch.uint8, device="cuda"), scalar(), scalar())
               for c in ref]
        full = [fp8.AdamChunk(c.g, c.g_inv, c.m, c.m_scale, c.v, c.v_scale, c.w, c.w_scale, None,
                              torch.empty(c.g.numel(), dtype=torch.uint8, device="cuda"), scalar(), scalar())
                for c in full]
    bounds = [[zero.shard_bounds(n, world, r) for n in sizes] for r in range(world)]
    ranks = [[zero.shard_chunk(c, lo, hi) for c, (lo, hi) in zip(full, bounds[r])] for r in range(world)]
    ws_ref = torch.zeros(fp8.fp8_adam_workspace_bytes(len(sizes)) // 4, **F32)
    ws = [torch.zeros_like(ws_ref) for _ in range(world)]
    ties = []
    for step in (1, 2):
        before = [snapshot(c) for c in ref]
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws_ref, **HP)
        for r in range(world):
            fp8.fp8_adam_stats(ranks[r], step=step, margin=0, workspace=ws[r], **HP)
        _reduce_max_int32(ws)
        for r in range(world):
            fp8.fp8_adam_apply(ranks[r], step=step, margin=0, workspace=ws[r], **HP)
        assert fp8.fp8_get_status() == 0
        for k, c in enumerate(ref):
            s = snapshot(c)
            for r in range(world):
                lo, hi = bounds[r][k]
                mine = ranks[r][k]
                assert (mine.m_scale.item(), mine.v_scale.item(), mine.w_scale.item()) == \
                    (s["s_m"], s["s_v"], s["s_w"]), (step, k, r)
                if wq:
                    assert (mine.wq_scale.item(), mine.wq_inv.item()) == (c.wq_scale.item(), c.wq_inv.item())
            # the slices are views of `full`, so the whole tensor can be compared at once
            f = snapshot(full[k])
            for key in ("m", "v", "w"):
                assert np.array_equal(f[key], s[key]), (step, k, key)
            if wq:
                assert torch.equal(full[k].wq, c.wq)
            if before[k]["g"].size:
                check_adam_chunk(before[k], c, step, ties=ties)
    assert len(ties) <= MAX_TIES, ties


def test_adam_sharded_halves_reject_tracking_and_bad_workspace():
    chunks = _with_tracking(make_adam_state([64], ("adam-shard-bad",)))
    ws = torch.zeros(16, **F32)
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_adam_stats(chunks, step=1, margin=0, workspace=ws, **HP)
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_adam_apply(chunks, step=1, margin=0, workspace=ws, **HP)
    plain = make_adam_state([64], ("adam-shard-bad",))
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_adam_stats(plain, step=1, margin=0, workspace=ws[:3], **HP)


def test_two_step_linear_chain_reads_adam_weight_copy():
    """f1 in a training chain: step 1 runs fwd/dgrad/wgrad on the E4M3 weight
    cast from the initial weights, casts the gradient (mu-scaled E5M2) and
    takes the Adam step, which also writes the E4M3 copy of the new master;
    step 2's fwd and dgrad read that copy and its inverse scale.  The copy
    equals the oracle's E4M3 cast of the stored master (codes and scale), and
    step 2's outputs match the oracle's GEMMs on it."""
    from fp8_mixed_precision_tensor_b200.adam_state import AdamTensorState, FP8Adam

    M, N, K = 512, 768, 1024
    W = to_dev(synth.normal_f32((N, K), 0.02, "chain", "W"))
    st = AdamTensorState(W, track_master_amax=True, e4m3_copy=True)
    opt = FP8Adam([st], **HP)
    wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    w_sc = torch.zeros(3, **F32)  # amax, scale, inverse of the step-1 weight operand
    fp8.fp8_amax(W, w_sc[0:1])
    fp8.fp8_scale_cast(W, fp8.FP8_E4M3, w_sc[0:1], 0, 1.0, w_sc[1:2], w_sc[2:3], wq)
    w_inv = w_sc[2:3]
    for step in (1, 2):
        X = to_dev(synth.normal_f32((M, K), 1.0, "chain", "X", step))
        dY = to_dev(synth.normal_f32((M, N), 1e-4, "chain", "dY", step))
        sc = torch.zeros(9, **F32)
        xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        dyq = torch.empty((M, N), dtype=torch.uint8, device="cuda")
        fp8.fp8_amax(X, sc[0:1])
        fp8.fp8_scale_cast(X, fp8.FP8_E4M3, sc[0:1], 0, 1.0, sc[1:2], sc[2:3], xq)
        fp8.fp8_amax(dY, sc[3:4])
        fp8.fp8_scale_cast(dY, fp8.FP8_E5M2, sc[3:4], 0, 2.0 ** 10, sc[4:5], sc[5:6], dyq)
        y = torch.empty((M, N), **F32)
        dx = torch.empty((M, K), **F32)
        dw = torch.empty((N, K), **F32)
        fp8.fp8_linear_fwd(xq, sc[2:3], wq if step == 1 else st.wq.view(N, K), w_inv, y)
        fp8.fp8_linear_dgrad(dyq, sc[5:6], wq if step == 1 else st.wq.view(N, K), w_inv, dx)
        fp8.fp8_linear_wgrad(dyq, sc[5:6], xq, sc[2:3], dw, sc[6:7])
        if step == 2:
            # the weight operand is the copy step 1's Adam wrote: check the GEMMs on it
            w_codes = st.wq.cpu().numpy().reshape(N, K)
            h_x, h_dy = xq.cpu().numpy(), dyq.cpu().numpy()
            ref, rabs = oracle.linear_fwd(h_x, sc[2].item(), w_codes, w_inv.item(), M, N, K)
            assert_gemm_close(tensor_to_np(y), ref, rabs, torch.float32, "step-2 fwd on the Adam copy")
            ref, rabs = oracle.linear_dgrad(h_dy, sc[5].item(), w_codes, w_inv.item(), M, N, K)
            assert_gemm_close(tensor_to_np(dx), ref, rabs, torch.float32, "step-2 dgrad on the Adam copy")
            break
        st.set_gradient(dw, 2.0 ** 10, grad_amax=sc[6:7])
        opt.step()
        assert fp8.fp8_get_status() == 0
        # the copy is the oracle's E4M3 cast of the stored FP16 master
        q_ref, s_q = oracle.adam_master_e4m3(st.w.cpu().numpy(), st.scalars[3].item(), 0)
        assert st.wq_scale.item() == s_q and st.wq_inv.item() == 1.0 / s_q
        assert np.array_equal(st.wq.cpu().numpy(), q_ref)
        w_inv = st.wq_inv
    assert fp8.fp8_get_status() == 0
