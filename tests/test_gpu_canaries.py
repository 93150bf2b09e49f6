"""Guard canaries around every output buffer of the C ABI.

Each output (codes, scales, amaxes, counters, GEMM outputs, Adam state and
its second buffers) is placed inside a larger device buffer whose bytes
before and after it -- 256 on each side, and the padding up to the next
16-byte boundary -- hold a fixed pattern.  After the call the pattern must be
intact: no kernel wrote outside its output, in particular not with a
16-byte vector store past a ragged end.  Sizes are small and odd (1, 15, 17,
4099, 65539 elements; GEMM shapes that are multiples of 16 but not of the
tile sizes, one per kernel the dispatcher picks).  Values are checked by the
parity tests; this file checks only where the kernels write.
"""
import numpy as np
import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8, synth

from test_gpu_parity import HP, _with_tracking, make_adam_state

pytestmark = pytest.mark.gpu

GUARD = 256
PATTERN = 0xA5
SIZES = [1, 15, 17, 4099, 65536 + 3]


class Guarded:
    """A device tensor of `numel` elements inside a guarded byte buffer."""

    def __init__(self, numel, dtype, init=None):
        item = torch.empty(0, dtype=dtype).element_size()
        self.nbytes = numel * item
        padded = (self.nbytes + 15) // 16 * 16
        self.raw = torch.full((GUARD + padded + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype)
        if init is not None:
            self.t.copy_(init.reshape(-1))

    def intact(self):
        r = self.raw.cpu().numpy()
        return bool((r[:GUARD] == PATTERN).all() and (r[GUARD + self.nbytes:] == PATTERN).all())


def _all_intact(**bufs):
    bad = [k for k, b in bufs.items() if not b.intact()]
    assert not bad, bad


def _f32(n=1, init=None):
    return Guarded(n, torch.float32, init)


DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


@pytest.mark.parametrize("dtype", list(DTYPES))
@pytest.mark.parametrize("n", SIZES)
def test_amax_scale_cast_family_writes_only_its_outputs(dtype, n):
    x = synth.device_normal((n,), 1.0, 1000 * n + DTYPES[dtype], dtype, "cuda")
    amax = _f32()
    fp8.fp8_amax(x, amax.t)
    for fmt in (fp8.FP8_E4M3, fp8.FP8_E5M2, fp8.FP8_F16S):
        qdt = torch.int16 if fmt == fp8.FP8_F16S else torch.uint8
        s, inv, q = _f32(), _f32(), Guarded(n, qdt)
        fp8.fp8_compute_scale(amax.t, fmt, 0, 1.0, s.t, inv.t)
        fp8.fp8_cast(x, fmt, s.t, q.t)
        s2, inv2, q2 = _f32(), _f32(), Guarded(n, qdt)
        fp8.fp8_scale_cast(x, fmt, amax.t, 1, 2.0 ** 4, s2.t, inv2.t, q2.t)
        a5, s5, inv5, q5 = _f32(), _f32(1, torch.tensor([0.5])), _f32(), Guarded(n, qdt)
        fp8.fp8_amax_scale_cast(x, fmt, a5.t, 0, 1.0, s5.t, inv5.t, q5.t)  # a wrong prediction: the redo runs
        a6, s6, inv6, q6 = _f32(), _f32(1, s5.t.cpu()), _f32(), Guarded(n, qdt)
        fp8.fp8_amax_scale_cast(x, fmt, a6.t, 0, 1.0, s6.t, inv6.t, q6.t)  # the right one: one pass
        _all_intact(amax=amax, s=s, inv=inv, q=q, s2=s2, inv2=inv2, q2=q2, a5=a5, s5=s5, inv5=inv5, q5=q5,
                    a6=a6, s6=s6, inv6=inv6, q6=q6)
        assert torch.equal(q5.t, q.t) and torch.equal(q6.t, q.t)
        if fmt != fp8.FP8_F16S:
            q3, counts = Guarded(n, torch.uint8), Guarded(2, torch.int64, torch.zeros(2, dtype=torch.int64))
            fp8.fp8_cast_count(x, fmt, s.t, q3.t, counts.t)
            mu = _f32(1, torch.tensor([2.0 ** 3]))
            s4, inv4, q4 = _f32(), _f32(), Guarded(n, torch.uint8)
            counts4 = Guarded(2, torch.int64, torch.zeros(2, dtype=torch.int64))
            fp8.fp8_grad_cast(x, fmt, amax.t, 0, mu.t, s4.t, inv4.t, q4.t, counts4.t)
            _all_intact(q3=q3, counts=counts, mu=mu, s4=s4, inv4=inv4, q4=q4, counts4=counts4)
            assert torch.equal(q3.t, q.t)


@pytest.mark.parametrize("n", [1, 17, 4099, 65536 + 3])
@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
def test_sum_codes_writes_only_its_outputs(n, fmt):
    nranks = 3
    ld = (n + 15) // 16 * 16
    g = torch.Generator(device="cpu").manual_seed(n)
    rows = torch.randint(0, 0x70, (nranks, ld), generator=g, dtype=torch.uint8).cuda()
    out, inv = Guarded(n, torch.uint8), _f32(1, torch.tensor([2.0 ** -10]))
    g_inv, counts = _f32(), Guarded(2, torch.int64, torch.zeros(2, dtype=torch.int64))
    fp8.fp8_sum_codes(rows, n, fmt, out.t, inv.t, g_inv.t, counts.t)
    _all_intact(out=out, inv=inv, g_inv=g_inv, counts=counts)


# one shape per GEMM kernel the dispatcher picks (one-CTA, pair, wide pair)
GEMM_SHAPES = [(272, 528, 80), (1040, 4112, 96), (2064, 4112, 64)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemms_write_only_their_outputs(M, N, K):
    g = torch.Generator(device="cpu").manual_seed(M + N + K)
    codes = lambda r, c: torch.randint(0, 0x70, (r, c), generator=g, dtype=torch.uint8).cuda()
    xq, wq, dyq = codes(M, K), codes(N, K), codes(M, N)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    y, ya = Guarded(M * N, torch.bfloat16), _f32()
    fp8.fp8_linear_fwd(xq, one, wq, one, y.t.view(M, N), ya.t)
    dx, dxa = Guarded(M * K, torch.bfloat16), _f32()
    fp8.fp8_linear_dgrad(dyq, one, wq, one, dx.t.view(M, K), dxa.t)
    dw, dwa = Guarded(N * K, torch.float32), _f32()
    fp8.fp8_linear_wgrad(dyq, one, xq, one, dw.t.view(N, K), dwa.t)
    dwr, dwra = Guarded(N * K, torch.bfloat16), _f32()
    fp8.fp8_linear_wgrad(dyq, one, xq, one, dwr.t.view(N, K), dwra.t, rto=True)
    y16, y16a = Guarded(M * N, torch.float16), _f32()
    fp8.fp8_linear_fwd(xq, one, wq, one, y16.t.view(M, N), y16a.t)
    assert fp8.fp8_get_status() == 0
    _all_intact(y=y, ya=ya, dx=dx, dxa=dxa, dw=dw, dwa=dwa, dwr=dwr, dwra=dwra, y16=y16, y16a=y16a)


def _guarded_adam_chunks(sizes, key):
    """Adam chunks whose every written buffer (m, v, w, scales, tracked amax,
    E4M3 copy and its scales) sits inside guards, seeded from make_adam_state."""
    src = _with_tracking(make_adam_state(sizes, key), wq=True)
    guards, chunks = [], []
    for c in src:
        n = c.g.numel()
        gm, gv, gw = Guarded(n, torch.uint8, c.m), Guarded(n, torch.int16, c.v), Guarded(n, torch.int16, c.w)
        sm, sv, sw = _f32(1, c.m_scale), _f32(1, c.v_scale), _f32(1, c.w_scale)
        wa, q, qs, qi = _f32(1, c.w_amax), Guarded(n, torch.uint8), _f32(), _f32()
        guards += [gm, gv, gw, sm, sv, sw, wa, q, qs, qi]
        chunks.append(fp8.AdamChunk(c.g, c.g_inv, gm.t, sm.t, gv.t, sv.t, gw.t, sw.t, wa.t, q.t, qs.t, qi.t))
    return chunks, guards


def test_adam_steps_write_only_their_outputs():
    sizes = [1, 17, 4099, 65536 + 5, 0]
    chunks, guards = _guarded_adam_chunks(sizes, ("canary-adam",))
    ws = Guarded(fp8.fp8_adam_workspace_bytes(len(sizes)) // 4, torch.float32)
    ws.t.zero_()
    for step in (1, 2):
        fp8.fp8_adam_step(chunks, step=step, margin=0, workspace=ws.t, **HP)
    dests = [(Guarded(c.g.numel(), torch.uint8), Guarded(c.g.numel(), torch.int16),
              Guarded(c.g.numel(), torch.int16)) for c in chunks]
    for step in (3, 4):  # the second set written, then the first again
        src = chunks if step == 3 else [fp8.AdamChunk(c.g, c.g_inv, m.t, c.m_scale, v.t, c.v_scale, w.t,
                                                      c.w_scale, c.w_amax, c.wq, c.wq_scale, c.wq_inv)
                                        for c, (m, v, w) in zip(chunks, dests)]
        dst = [(m.t, v.t, w.t) for m, v, w in dests] if step == 3 else [(c.m, c.v, c.w) for c in chunks]
        fp8.fp8_adam_step_into(src, dst, step=step, margin=0, workspace=ws.t, **HP)
    # step 5 with the gradient cast in the pass (bf16 gradients): writes the first set again
    dws = [torch.full((c.g.numel(),), 1e-3, dtype=torch.bfloat16, device="cuda") for c in chunks]
    amax = [_f32(1, torch.tensor([1e-3])) for _ in chunks]
    ginv = [_f32() for _ in chunks]
    src = [fp8.AdamChunk(dw, gi.t, m.t, c.m_scale, v.t, c.v_scale, w.t, c.w_scale, None, c.wq, c.wq_scale,
                         c.wq_inv) for c, dw, gi, (m, v, w) in zip(chunks, dws, ginv, dests)]
    fp8.fp8_adam_step_into_castgrad(src, [(c.m, c.v, c.w) for c in chunks], [a.t for a in amax], 1024.0, 0,
                                    step=5, margin=0, workspace=ws.t, **HP)
    assert fp8.fp8_get_status() == 0
    assert all(g.intact() for g in guards)
    assert all(b.intact() for d in dests for b in d)
    assert all(g.intact() for g in ginv + amax)
    assert ws.intact()
