"""Run one kernel family of the hot path on a chosen case (for profilers).

    python profile_cases.py linear --M 4096 --N 16384 --K 4096 [--rto]
    python profile_cases.py cast --n 268435456 [--onepass]
    python profile_cases.py castsweep
    python profile_cases.py adam --n 67108864 [--track] [--into]
    python profile_cases.py allreduce --n 268435456 --world 8
    python profile_cases.py castcount --n 268435456
    python profile_cases.py adam7b --iters 10 [--track] [--copy] [--into]

Each case runs `--iters` passes after one warm-up pass (and `--skip` more) on
seeded synthetic inputs and prints the CUDA-event time per pass.  Launch order per pass:
linear: amax and fused scale+cast of X, W, dY (6 launches), then fwd, dgrad,
wgrad; cast: amax, fused scale+cast; adam: stats pass, finalize, update pass
(with --into the out-of-place step: update with the predicted scales,
finalize, redo pass, finalize);
allreduce: `world` emulated ranks' payload casts of an fp32 gradient, then
the `world` per-slice code sums (no collective: one GPU); castcount: the cast
with under/overflow counters, then the plain cast; adam7b: one Adam step
over all 129 per-tensor chunks of GPT-7B (6,648,496,128 parameters, 40 GB
of FP8/FP16 state).  allreduce, castcount and adam7b also print each
kernel's own time and algorithmic GB/s.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from fp8_mixed_precision_tensor_b200 import fp8, synth  # noqa: E402
from fp8_mixed_precision_tensor_b200.adam_state import AdamTensorState, FP8Adam  # noqa: E402


def _scalars(n):
    return torch.zeros(n, dtype=torch.float32, device="cuda")


def case_linear(a):
    M, N, K = a.M, a.N, a.K
    X = synth.device_normal((M, K), synth.ACT_STD, 1, torch.bfloat16, "cuda")
    W = synth.device_normal((N, K), synth.GPT7B_W_STD, 2, torch.bfloat16, "cuda")
    dY = synth.device_normal((M, N), synth.GRAD_STD, 3, torch.bfloat16, "cuda")
    u8 = dict(dtype=torch.uint8, device="cuda")
    xq, wq, dyq = torch.empty((M, K), **u8), torch.empty((N, K), **u8), torch.empty((M, N), **u8)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    # --rto: dW as bfloat16 rounded to odd (the bench step's form), else float32
    dw = torch.empty((N, K), dtype=torch.bfloat16 if a.rto else torch.float32, device="cuda")
    sc = _scalars(16)

    def one():
        for t, q, i, fmt in ((X, xq, 0, fp8.FP8_E4M3), (W, wq, 3, fp8.FP8_E4M3), (dY, dyq, 6, fp8.FP8_E5M2)):
            fp8.fp8_amax(t, sc[i:i + 1])
            fp8.fp8_scale_cast(t, fmt, sc[i:i + 1], 0, 1.0, sc[i + 1:i + 2], sc[i + 2:i + 3], q)
        fp8.fp8_linear_fwd(xq, sc[2:3], wq, sc[5:6], y, sc[12:13])
        fp8.fp8_linear_dgrad(dyq, sc[8:9], wq, sc[5:6], dx, sc[13:14])
        fp8.fp8_linear_wgrad(dyq, sc[8:9], xq, sc[2:3], dw, sc[14:15], rto=a.rto)

    one()
    flops = 2.0 * M * N * K
    for name, fn in (("fwd", lambda: fp8.fp8_linear_fwd(xq, sc[2:3], wq, sc[5:6], y, sc[12:13])),
                     ("dgrad", lambda: fp8.fp8_linear_dgrad(dyq, sc[8:9], wq, sc[5:6], dx, sc[13:14])),
                     ("wgrad", lambda: fp8.fp8_linear_wgrad(dyq, sc[8:9], xq, sc[2:3], dw, sc[14:15], rto=a.rto))):
        t = _timed(fn, max(a.iters, 3))
        print(f"  {name:5s} M{M} N{N} K{K}: {t:.4f} ms, {flops / t / 1e9:.1f} TFLOP/s")
    return one


def case_cast(a):
    x = synth.device_normal((a.n,), 1.0, 4, torch.bfloat16, "cuda")
    q = torch.empty(a.n, dtype=torch.uint8, device="cuda")
    sc = _scalars(3)

    def one():
        if a.onepass:  # amax, scale and cast reading x once (the scale of the previous pass as the guess)
            fp8.fp8_amax_scale_cast(x, fp8.FP8_E4M3, sc[0:1], 0, 1.0, sc[1:2], sc[2:3], q)
        else:
            fp8.fp8_amax(x, sc[0:1])
            fp8.fp8_scale_cast(x, fp8.FP8_E4M3, sc[0:1], 0, 1.0, sc[1:2], sc[2:3], q)

    return one


def case_castsweep(a):
    """amax + fused scale/cast of bf16 tensors of 2^20..2^28 elements to E4M3
    and E5M2, margin 0 and 1: device time per pass from a CUDA-graph replay,
    GB/s (2 B amax read + 2 B read + 1 B write per element), and the time when
    the two calls are issued one by one from Python."""
    big = synth.device_normal((1 << 28,), 1.0, 4, torch.bfloat16, "cuda")
    qbuf = torch.empty(1 << 28, dtype=torch.uint8, device="cuda")
    sc = _scalars(3)
    for e in range(20, 29, 2):
        n = 1 << e
        x, q = big[:n], qbuf[:n]
        for fmt in (fp8.FP8_E4M3, fp8.FP8_E5M2):
            for margin in (0, 1):
                def f():
                    fp8.fp8_amax(x, sc[0:1])
                    fp8.fp8_scale_cast(x, fmt, sc[0:1], margin, 1.0, sc[1:2], sc[2:3], q)
                # replay 20 passes captured in a CUDA graph: device time without
                # the per-call host cost that dominates the small sizes
                f()
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    for _ in range(20):
                        f()
                t = _timed(graph.replay, 3) / 20
                t_host = _timed(f, 20)
                print(f"  2^{e} fmt {fmt} margin {margin}: {t * 1e3:8.1f} us, {5 * n / t / 1e6:7.0f} GB/s "
                      f"(graph replay; issued call by call: {t_host * 1e3:.1f} us)")

    def one():
        fp8.fp8_amax(big, sc[0:1])
        fp8.fp8_scale_cast(big, fp8.FP8_E4M3, sc[0:1], 0, 1.0, sc[1:2], sc[2:3], qbuf)

    return one


def case_adam(a):
    n = a.n
    g = synth.device_normal((n,), 1e-3, 5, torch.float32, "cuda")
    w = synth.device_normal((n,), 0.02, 6, torch.float32, "cuda")
    sc = _scalars(8)
    gq = torch.empty(n, dtype=torch.uint8, device="cuda")
    wh = torch.empty(n, dtype=torch.int16, device="cuda")
    fp8.fp8_amax(g, sc[0:1])
    fp8.fp8_compute_scale(sc[0:1], fp8.FP8_E5M2, 0, 2.0 ** 10, sc[1:2], sc[2:3])
    fp8.fp8_cast(g, fp8.FP8_E5M2, sc[1:2], gq)
    fp8.fp8_amax(w, sc[3:4])
    fp8.fp8_compute_scale(sc[3:4], fp8.FP8_F16S, 0, 1.0, sc[4:5], sc[5:6])
    fp8.fp8_cast(w, fp8.FP8_F16S, sc[4:5], wh)
    del g, w
    m = torch.zeros(n, dtype=torch.uint8, device="cuda")
    v = torch.zeros(n, dtype=torch.int16, device="cuda")
    st = torch.ones(3, dtype=torch.float32, device="cuda")
    st[2] = -1.0  # tracked master amax: unknown until the first step
    bufs = [(m, v, wh)]
    if a.into:
        bufs.append((torch.empty_like(m), torch.empty_like(v), torch.empty_like(wh)))
    packs = [(fp8.pack_adam_chunks([fp8.AdamChunk(gq, sc[2:3], mm, st[0:1], vv, st[1:2], ww, sc[4:5],
                                                  w_amax=st[2:3] if a.track else None)]),
              fp8.pack_adam_dests([bufs[1 - k]]) if a.into else None)
             for k, (mm, vv, ww) in enumerate(bufs)]
    ws = torch.zeros(64, dtype=torch.float32, device="cuda")
    state = {"t": 0}

    def one():
        state["t"] += 1
        chunks, dests = packs[(state["t"] - 1) % len(packs)]
        if a.into:
            fp8.fp8_adam_step_into(chunks, dests, 1e-4, 0.9, 0.95, 1e-8, state["t"], 0, ws)
        else:
            fp8.fp8_adam_step(chunks, 1e-4, 0.9, 0.95, 1e-8, state["t"], 0, ws)

    return one


def _timed(fn, iters):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()
    s.record()
    for _ in range(iters):
        fn()
    e.record()
    e.synchronize()
    return s.elapsed_time(e) / iters


def case_allreduce(a):
    n, world = a.n, a.world
    L = -(-(-(-n // 16)) // world) * 16
    g = synth.device_normal((n,), 1e-4, 7, torch.float32, "cuda")
    amax, mu, sc = _scalars(1), torch.full((1,), 1.0 / world, device="cuda"), _scalars(3)
    fp8.fp8_amax(g, amax)
    sends = torch.zeros(world, world * L, dtype=torch.uint8, device="cuda")
    out = torch.zeros(world * L, dtype=torch.uint8, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    rows = torch.zeros(world, L, dtype=torch.uint8, device="cuda")

    def casts():
        for r in range(world):
            fp8.fp8_grad_cast(g, fp8.FP8_E5M2, amax, 0, mu, sc[0:1], sc[1:2], sends[r], counts)

    def sums():
        for j in range(world):
            fp8.fp8_sum_codes(rows, L, fp8.FP8_E5M2, out[j * L:(j + 1) * L], sc[1:2], sc[2:3], counts)

    casts()
    rows.copy_(sends[:, :L])
    t_cast = _timed(casts, a.iters) / world
    t_sum = _timed(sums, a.iters) / world
    print(f"grad_cast: {t_cast:.4f} ms per rank, {5 * n / t_cast / 1e6:.0f} GB/s (4 B read + 1 B write per elem)")
    print(f"sum_codes: {t_sum:.4f} ms per slice, {(world + 1) * L / t_sum / 1e6:.0f} GB/s "
          f"({world} B read + 1 B write per slice elem)")

    def one():
        casts()
        sums()

    return one


def case_castcount(a):
    x = synth.device_normal((a.n,), 1.0, 8, torch.bfloat16, "cuda")
    q = torch.empty(a.n, dtype=torch.uint8, device="cuda")
    s = torch.full((1,), 2.0 ** 6, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    t_count = _timed(lambda: fp8.fp8_cast_count(x, fp8.FP8_E4M3, s, q, counts), a.iters)
    t_plain = _timed(lambda: fp8.fp8_cast(x, fp8.FP8_E4M3, s, q), a.iters)
    print(f"cast_count: {t_count:.4f} ms, {3 * a.n / t_count / 1e6:.0f} GB/s; plain cast: {t_plain:.4f} ms, "
          f"{3 * a.n / t_plain / 1e6:.0f} GB/s (2 B read + 1 B write per elem)")

    def one():
        fp8.fp8_cast_count(x, fp8.FP8_E4M3, s, q, counts)
        fp8.fp8_cast(x, fp8.FP8_E4M3, s, q)

    return one


def build_adam_state(chunks, device="cuda", seed=11, mu=2.0 ** 10, track=False, copy=False, spare=False):
    """Decoupled-Adam state for (name, n) chunks: FP16 master from weights
    ~N(0, 0.02), zero moments, E5M2 gradients ~N(0, 1e-3) scaled by mu; with
    `copy` the step also writes each tensor's E4M3 weight copy, with `spare`
    each state gets the out-of-place step's second buffers.  Returns the
    AdamTensorState list."""
    out = []
    for ci, (_, n) in enumerate(chunks):
        w = synth.device_normal((n,), 0.02, seed * 100000 + 2 * ci + 1, torch.float32, device)
        st = AdamTensorState(w, track_master_amax=track, e4m3_copy=copy, spare_buffers=spare)
        del w
        g = synth.device_normal((n,), 1e-3, seed * 100000 + 2 * ci, torch.float32, device)
        st.set_gradient(g, mu)
        del g
        out.append(st)
    return out


def case_adam7b(a):
    states = build_adam_state(synth.gpt7b_adam_chunks(), track=a.track, copy=a.copy, spare=a.into)
    opt = FP8Adam(states, lr=1e-4, out_of_place=a.into)
    params = sum(st.n for st in states)

    def one():
        opt.step()

    t = _timed(one, a.iters)
    # bytes moved per parameter: the stats pass reads g, m, v (and the master
    # unless its amax is tracked), the update pass reads g, m, v, w and writes
    # m, v, w (and the E4M3 copy); out of place, the update pass alone (while
    # the scales hold)
    moved = (0 if a.into else (4 if a.track else 6)) + 11 + (1 if a.copy else 0)
    print(f"adam7b: {len(states)} chunks, {params} params, track={a.track} copy={a.copy} into={a.into}: "
          f"{t:.3f} ms per step, {11 * params / t / 1e6:.0f} GB/s algorithmic (11 B/param), "
          f"{moved * params / t / 1e6:.0f} GB/s moved ({moved} B/param)")
    return one


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["linear", "cast", "castsweep", "adam", "allreduce", "castcount", "adam7b"])
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=16384)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--n", type=int, default=1 << 26)
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--world", type=int, default=8, help="allreduce: emulated ranks")
    ap.add_argument("--track", action="store_true", help="adam: track the master amax across steps")
    ap.add_argument("--copy", action="store_true", help="adam7b: write the E4M3 weight copy")
    ap.add_argument("--into", action="store_true", help="adam, adam7b: the out-of-place step")
    ap.add_argument("--skip", type=int, default=0,
                    help="passes run before the timed ones besides the one warm-up pass (adam: steps "
                         "after which the moments' scales have settled)")
    ap.add_argument("--rto", action="store_true", help="linear: dW as bfloat16 rounded to odd")
    ap.add_argument("--onepass", action="store_true", help="cast: amax, scale and cast in one call")
    a = ap.parse_args()
    one = {"linear": case_linear, "cast": case_cast, "castsweep": case_castsweep, "adam": case_adam,
           "allreduce": case_allreduce,
           "castcount": case_castcount, "adam7b": case_adam7b}[a.case](a)
    for _ in range(1 + a.skip):
        one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(a.iters):
        one()
    e.record()
    e.synchronize()
    status = fp8.fp8_get_status()
    print(f"{a.case}: {s.elapsed_time(e) / a.iters:.4f} ms per pass, device status {status}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
