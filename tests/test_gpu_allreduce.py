"""Scaling variants and the FP8 gradient all-reduce on the GPU vs the oracle
("FP8-LM", 提案手法 O1 with Eq. 3 and アブレーション研究; "Training and
inference of large language models using 8-bit floating point", 실험 결과,
FP8-CSCALE against FP8-AMAX).

Bars: codes, scales and under/overflow counts bit-exact; the mu rule's state
equal step by step.  Several ranks are emulated one after another on this
GPU: their kernels never wait on one another, and the exchange between them
is a device copy in the layout the all-to-all produces."""
import numpy as np
import pytest
import torch

import oracle
from fp8_mixed_precision_tensor_b200 import fp8, synth, zero
from _util import assert_codes_equal, bf16_dev, to_dev

pytestmark = pytest.mark.gpu

F32 = dict(dtype=torch.float32, device="cuda")
I64 = dict(dtype=torch.int64, device="cuda")
ODT = {fp8.FP8_DT_F32: oracle.DT_F32, fp8.FP8_DT_BF16: oracle.DT_BF16}
OFMT = {fp8.FP8_E4M3: oracle.E4M3, fp8.FP8_E5M2: oracle.E5M2, fp8.FP8_F16S: oracle.F16}


def _input(n, dt, key):
    b = synth.lognormal_outliers_bf16(n, *key)
    x = synth.bf16_bits_to_f32(b).copy()
    if n >= 16:
        x[[2, 5, n - 1]] = [np.inf, np.nan, -0.0]
        x[7] = 1e-30
    if dt == fp8.FP8_DT_F32:
        return x, to_dev(x)
    bits = synth.to_bf16_bits(x)
    return bits, bf16_dev(bits)


@pytest.mark.parametrize("dt", [fp8.FP8_DT_F32, fp8.FP8_DT_BF16])
@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2, fp8.FP8_F16S])
@pytest.mark.parametrize("bias", [-8, 0, 6, 12])
def test_cast_count_constant_scale_vs_oracle(dt, fmt, bias):
    """FP8-CSCALE: a constant scaling bias 2^bias instead of the amax rule;
    the counts show what it loses (log-normal data spans ~2^-20..2^13)."""
    n = (1 << 18) + 11
    h, d = _input(n, dt, ("ccount", dt, fmt, bias))
    s = torch.full((1,), 2.0 ** bias, **F32)
    q = torch.empty(n, dtype=torch.int16 if fmt == fp8.FP8_F16S else torch.uint8, device="cuda")
    counts = torch.zeros(2, **I64)
    fp8.fp8_cast_count(d, fmt, s, q, counts)
    ref, rc = oracle.cast_counts(h, OFMT[fmt], 2.0 ** bias, ODT[dt])
    got = q.cpu().numpy()
    xin = h if dt == fp8.FP8_DT_F32 else synth.bf16_bits_to_f32(h)
    assert_codes_equal(got.view(np.uint16) if fmt == fp8.FP8_F16S else got, ref, xin, "cast_count")
    assert tuple(counts.tolist()) == rc
    # the plain cast writes the same codes
    q2 = torch.empty_like(q)
    fp8.fp8_cast(d, fmt, s, q2)
    assert torch.equal(q, q2)
    # counts accumulate
    fp8.fp8_cast_count(d, fmt, s, q, counts)
    assert tuple(counts.tolist()) == (2 * rc[0], 2 * rc[1])


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
@pytest.mark.parametrize("mu,margin", [(1.0, 0), (2.0 ** -3, 0), (2.0 ** -2, 1), (4.0, 0)])
def test_grad_cast_vs_oracle(fmt, mu, margin):
    n = (1 << 17) + 5
    g = synth.normal_f32((n,), 1e-3, "gcast", fmt, mu, margin)
    g[9] = 0.02
    d = to_dev(g)
    amax = torch.full((1,), 0.05, **F32)  # the amax over all ranks, larger than this rank's
    mu_d = torch.full((1,), mu, **F32)
    S, inv = torch.zeros(1, **F32), torch.zeros(1, **F32)
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    counts = torch.zeros(2, **I64)
    fp8.fp8_grad_cast(d, fmt, amax, margin, mu_d, S, inv, q, counts)
    rc, S_ref = oracle.grad_scale(float(np.float32(0.05)), OFMT[fmt], margin, mu)
    assert S.item() == S_ref and inv.item() == 1.0 / S_ref
    ref, c = oracle.cast_counts(g, OFMT[fmt], S_ref)
    assert_codes_equal(q.cpu().numpy(), ref, g, "grad_cast")
    assert tuple(counts.tolist()) == c
    assert fp8.fp8_get_status() == 0


def test_grad_cast_bad_mu_and_empty():
    n = 4096
    d = to_dev(synth.normal_f32((n,), 1.0, "gcast-bad"))
    amax = torch.full((1,), 2.0, **F32)
    S, inv = torch.zeros(1, **F32), torch.zeros(1, **F32)
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    fp8.fp8_grad_cast(d, fp8.FP8_E5M2, amax, 0, torch.full((1,), 3.0, **F32), S, inv, q)
    assert fp8.fp8_get_status() == fp8.FP8_STATUS_BAD_MU
    assert S.item() == oracle.grad_scale(2.0, oracle.E5M2, 0, 1.0)[1]
    S.zero_()
    fp8.fp8_grad_cast(torch.empty(0, **F32), fp8.FP8_E5M2, amax, 0, torch.full((1,), 0.5, **F32), S, inv,
                      torch.empty(0, dtype=torch.uint8, device="cuda"))
    assert S.item() == oracle.grad_scale(2.0, oracle.E5M2, 0, 0.5)[1]
    with pytest.raises(fp8.FP8Error):  # FP16 is not a payload format
        fp8.fp8_grad_cast(d, fp8.FP8_F16S, amax, 0, torch.ones(1, **F32), S, inv, q)


def _codes_with_specials(nranks, ld, fmt, key):
    c = synth.rng("sumcodes", *key).integers(0, 256, size=(nranks, ld), dtype=np.uint8)
    nan = (c & 0x7F) == 0x7F if fmt == fp8.FP8_E4M3 else (c & 0x7C) == 0x7C
    c[nan & (synth.rng("sumcodes-keep", *key).random(c.shape) > 0.002)] &= 0x83
    return c


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
@pytest.mark.parametrize("nranks", [1, 2, 3, 8])
@pytest.mark.parametrize("n", [16, 4099, (1 << 16) + 5])
def test_sum_codes_vs_oracle(fmt, nranks, n):
    ld = -(-n // 16) * 16 + 32
    rows = _codes_with_specials(nranks, ld, fmt, (fmt, nranks, n))
    if n > 8 and fmt == fp8.FP8_E5M2 and nranks > 1:  # +inf with -inf, +inf alone
        rows[0, 3], rows[1, 3] = 0x7C, 0xFC
        rows[:, 4] = 0x00
        rows[0, 4] = 0x7C
    d = to_dev(rows)
    out = torch.full((ld,), 0xAA, dtype=torch.uint8, device="cuda")
    inv = torch.full((1,), 2.0 ** -13, **F32)
    g_inv = torch.zeros(1, **F32)
    counts = torch.zeros(2, **I64)
    fp8.fp8_sum_codes(d, n, fmt, out, inv, g_inv, counts)
    ref, c = oracle.sum_codes(rows[:, :n], OFMT[fmt])
    got = out.cpu().numpy()
    assert_codes_equal(got[:n], ref, None, "sum_codes")
    assert np.all(got[n:] == 0xAA)  # nothing written past n
    assert tuple(counts.tolist()) == c
    assert g_inv.item() == float(np.float32(2.0 ** -13) * np.float32(1.0 / nranks))


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
def test_sum_codes_many_ranks(fmt):
    """160 ranks: E5M2 beyond the split-accumulator path's 128 ranks takes the
    integer path; E4M3 stays on the split path."""
    nranks, n = 160, 4099
    ld = -(-n // 16) * 16
    rows = _codes_with_specials(nranks, ld, fmt, ("many", fmt))
    out = torch.zeros(ld, dtype=torch.uint8, device="cuda")
    counts = torch.zeros(2, **I64)
    fp8.fp8_sum_codes(to_dev(rows), n, fmt, out, counts=counts)
    ref, c = oracle.sum_codes(rows[:, :n], OFMT[fmt])
    assert_codes_equal(out.cpu().numpy()[:n], ref, None, "sum_codes many ranks")
    assert tuple(counts.tolist()) == c


def test_sum_codes_rejects_bad_layout():
    d = torch.zeros(2, 40, dtype=torch.uint8, device="cuda")
    out = torch.zeros(48, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8.FP8Error):  # ld not a multiple of 16
        fp8.fp8_sum_codes(d, 32, fp8.FP8_E5M2, out)
    with pytest.raises(fp8.FP8Error):  # n > ld
        fp8.fp8_sum_codes(torch.zeros(2, 32, dtype=torch.uint8, device="cuda"), 48, fp8.FP8_E5M2, out)


def test_mu_update_vs_oracle_sequence():
    mu = torch.ones(1, **F32)
    clean = torch.zeros(1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, **I64)
    rule = dict(theta=1e-3, interval=3, mu_min=2.0 ** -4, mu_max=2.0)
    m_ref, c_ref = 1.0, 0
    for over in (0, 0, 0, 0, 0, 0, 2, 1, 5000, 5000, 5000, 5000, 5000, 0):
        counts.copy_(torch.tensor([7, over]))
        fp8.fp8_mu_update(mu, clean, counts, 1000, **rule)
        m_ref, c_ref = oracle.mu_update(m_ref, c_ref, over, 1000, float(np.float32(1e-3)), 3, 2.0 ** -4, 2.0)
        assert (mu.item(), clean.item()) == (m_ref, c_ref)
        assert counts.tolist() == [0, 0]
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_mu_update(mu, clean, counts, 1000, theta=1e-3, interval=3, mu_min=3.0, mu_max=4.0)


@pytest.mark.parametrize("scaling", ["post", "pre", "auto"])
@pytest.mark.parametrize("world", [2, 4])
def test_fp8_allreduce_emulated_ranks_vs_oracle(world, scaling):
    """The whole all-reduce for `world` ranks on one GPU: per-rank amax, the
    MAX over ranks, the payload cast, the all-to-all as a device copy, the
    per-slice sums; compared with the oracle's all-reduce, over three steps of
    the mu rule for "auto"."""
    n = 3 * 65536 + 77
    L = -(-(-(-n // 16)) // world) * 16
    mu_host = {"post": 1.0, "pre": 1.0 / world, "auto": 1.0}[scaling]
    mu = torch.full((1,), mu_host, **F32)
    clean = torch.zeros(1, dtype=torch.int32, device="cuda")
    clean_ref = 0
    for step in range(3):
        grads = []
        for r in range(world):
            g = synth.normal_f32((n,), 1e-4, "ar-gpu", world, step, r)
            g[:64] = np.float32(0.5 + 0.01 * r)   # same sign on all ranks: overflows at mu = 1
            g[100:116] = np.float32(2.0 ** -33)  # underflows when pre-divided
            grads.append(g)
        dev = [to_dev(g) for g in grads]
        amaxes = [torch.zeros(1, **F32) for _ in range(world)]
        for g, a in zip(dev, amaxes):
            fp8.fp8_amax(g, a)
        shared = torch.stack([a.view(torch.int32) for a in amaxes]).amax(0).view(torch.float32)
        S, inv = torch.zeros(1, **F32), torch.zeros(1, **F32)
        sends = [torch.zeros(world * L, dtype=torch.uint8, device="cuda") for _ in range(world)]
        cast_counts = torch.zeros(2, **I64)
        for r in range(world):
            fp8.fp8_grad_cast(dev[r], fp8.FP8_E5M2, shared, 0, mu, S, inv, sends[r], cast_counts)
        sum_counts = torch.zeros(2, **I64)
        out = torch.zeros(world * L, dtype=torch.uint8, device="cuda")
        g_inv = torch.zeros(1, **F32)
        for j in range(world):
            lo, hi = zero.shard_bounds(n, world, j)
            recv = torch.stack([sends[r][j * L:(j + 1) * L] for r in range(world)])
            fp8.fp8_sum_codes(recv, hi - lo, fp8.FP8_E5M2, out[lo:lo + L], inv, g_inv, sum_counts)
        want = oracle.fp8_allreduce(grads, oracle.E5M2, 0, mu_host)
        assert S.item() == want["S"]
        assert_codes_equal(out[:n].cpu().numpy(), want["codes"], None, "allreduce")
        assert tuple(cast_counts.tolist()) == want["cast_counts"]
        assert tuple(sum_counts.tolist()) == want["sum_counts"]
        if scaling == "post":
            assert want["sum_counts"][1] >= 64
        if scaling == "pre":
            assert want["cast_counts"][0] >= 16 * world
        if scaling == "auto":
            fp8.fp8_mu_update(mu, clean, sum_counts, n, theta=0.0, interval=2, mu_min=2.0 ** -16, mu_max=1.0)
            mu_host, clean_ref = oracle.mu_update(mu_host, clean_ref, want["sum_counts"][1], n, 0.0, 2,
                                                  2.0 ** -16, 1.0)
            assert (mu.item(), clean.item()) == (mu_host, clean_ref)
    assert fp8.fp8_get_status() == 0
