"""Full-size parity at the workloads' own shapes, in the launch configuration
the benchmark times: the GPT-7B and GPT-175B block linears (fwd, dgrad,
wgrad through the amax -> scale -> cast chain).  The oracle computes sampled
outputs one by one (random positions plus every tile edge); the fused output
amax is checked as a property that holds at any size (it equals the maximum
magnitude of the stored output)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_mixed_precision_tensor_b200 import fp8, synth
from _util import assert_gemm_close, boundary_samples, tensor_to_np

pytestmark = pytest.mark.gpu

F32 = dict(dtype=torch.float32, device="cuda")


def _quantise(t, fmt, mu=1.0):
    a, s, inv = (torch.zeros(1, **F32) for _ in range(3))
    q = torch.empty(t.shape, dtype=torch.uint8, device="cuda")
    fp8.fp8_amax(t, a)
    fp8.fp8_compute_scale(a, fmt, 0, mu, s, inv)
    fp8.fp8_cast(t, fmt, s, q)
    return q, s, inv, a


def _check_linear(M, K, N, w_std, seed):
    X = synth.device_normal((M, K), synth.ACT_STD, seed + 1, torch.bfloat16, "cuda")
    W = synth.device_normal((N, K), w_std, seed + 2, torch.bfloat16, "cuda")
    dY = synth.device_normal((M, N), synth.GRAD_STD, seed + 3, torch.bfloat16, "cuda")
    (xq, sx, xi, xa), (wq, sw, wi, wa), (dyq, sdy, dyi, dya) = (
        _quantise(X, fp8.FP8_E4M3), _quantise(W, fp8.FP8_E4M3), _quantise(dY, fp8.FP8_E5M2, 2.0 ** 10))
    # the scales are the oracle's for the amax the GPU found, and the amax is exact
    for t, a, s, fmt, mu in ((X, xa, sx, oracle.E4M3, 1.0), (W, wa, sw, oracle.E4M3, 1.0),
                             (dY, dya, sdy, oracle.E5M2, 2.0 ** 10)):
        assert a.item() == t.abs().max().float().item()
        assert s.item() == oracle.compute_scale(a.item(), fmt, 0, mu=mu)[1]
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ya, dxa, dwa = (torch.zeros(1, **F32) for _ in range(3))
    fp8.fp8_linear_fwd(xq, xi, wq, wi, y, ya)
    fp8.fp8_linear_dgrad(dyq, dyi, wq, wi, dx, dxa)
    fp8.fp8_linear_wgrad(dyq, dyi, xq, xi, dw, dwa)
    assert fp8.fp8_get_status() == 0
    xh, wh, dyh = xq.cpu().numpy(), wq.cpu().numpy(), dyq.cpu().numpy()
    for name, out, amax, (rows, cols), fn in (
            ("fwd", y, ya, (M, N), lambda s: oracle.linear_fwd(xh, xi.item(), wh, wi.item(), M, N, K, samples=s)),
            ("dgrad", dx, dxa, (M, K), lambda s: oracle.linear_dgrad(dyh, dyi.item(), wh, wi.item(), M, N, K,
                                                                     samples=s)),
            ("wgrad", dw, dwa, (N, K), lambda s: oracle.linear_wgrad(dyh, dyi.item(), xh, xi.item(), M, N, K,
                                                                     samples=s))):
        r, c = boundary_samples(rows, cols, 2000, (name, M, N, K), tile_c=(256, 512))
        ref, rabs = fn((r, c))
        got = tensor_to_np(out[torch.from_numpy(r).cuda(), torch.from_numpy(c).cuda()].contiguous())
        assert_gemm_close(got, ref, rabs, out.dtype, f"{name} M{M} N{N} K{K}")
        assert amax.item() == out.abs().max().float().item(), name
    del X, W, dY, y, dx, dw


@pytest.mark.parametrize("name,K,N", synth.GPT7B_LINEARS)
def test_gpt7b_linears_full_size(name, K, N):
    _check_linear(synth.GPT7B_TOKENS, K, N, synth.GPT7B_W_STD, 100)


@pytest.mark.parametrize("fmt,std", [(fp8.FP8_E4M3, synth.ACT_STD), (fp8.FP8_E5M2, synth.GRAD_STD)])
def test_one_pass_cast_at_the_largest_step_tensor(fmt, std):
    """The GPT-175B step's largest activation / output gradient (8192 x 49152
    bf16, 403 M elements): the one-pass amax + cast the benchmark runs gives
    the amax, scales and codes of the amax pass and fused scale + cast, bit
    for bit, with its guess right (one pass) and wrong (the redo)."""
    M, K = synth.GPT175B_TOKENS, 49152
    x = synth.device_normal((M, K), std, 4242 + fmt, torch.bfloat16, "cuda")
    mu = 2.0 ** 10 if fmt == fp8.FP8_E5M2 else 1.0
    f32 = dict(dtype=torch.float32, device="cuda")
    a, s, inv = (torch.zeros(1, **f32) for _ in range(3))
    q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    fp8.fp8_amax(x, a)
    fp8.fp8_scale_cast(x, fmt, a, 0, mu, s, inv, q)
    for guess in (s.item(), s.item() * 2.0):
        a1, inv1 = torch.zeros(1, **f32), torch.zeros(1, **f32)
        s1 = torch.full((1,), guess, **f32)
        q1 = torch.empty_like(q)
        fp8.fp8_amax_scale_cast(x, fmt, a1, 0, mu, s1, inv1, q1)
        assert (a1.item(), s1.item(), inv1.item()) == (a.item(), s.item(), inv.item()), guess
        assert torch.equal(q1, q), guess
    assert fp8.fp8_get_status() == 0
    del x, q, q1
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,K,N", synth.GPT175B_LINEARS)
def test_gpt175b_linears_full_size(name, K, N):
    _check_linear(synth.GPT175B_TOKENS, K, N, synth.GPT175B_W_STD, 200)


@pytest.mark.parametrize("workload", ["gpt7b_block", "gpt175b_block"])
def test_bench_step_three_streams_equals_one_stream(workload):
    """The benchmark step's overlapped schedule (casts, fwd/dgrad and wgrad on
    three streams, each tensor's Adam beside the next linears) computes exactly
    what the one-stream order computes, and the out-of-place Adam step (with
    the gradient cast kernel, and with the cast in its pass) exactly what the
    in-place step computes: the same scalars, gradient codes, Adam state and
    E4M3 weight copies after three steps (the second and third
    steps' GEMMs read the weights that the previous step's Adam wrote; out of
    place, the state after step 3 is in the second buffer set)."""
    import importlib.util
    import os

    spec = importlib.util.spec_from_file_location(
        "bench_mod", os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    dev = torch.device("cuda", 0)
    a = bench.BlockStep(dev, seed=3, workload=workload, adam="in_place")
    b = bench.BlockStep(dev, seed=3, workload=workload, adam="into")
    c = bench.BlockStep(dev, seed=3, workload=workload, adam="into", grad_cast="fused")
    for _ in range(3):
        a.step()
        b.step_overlapped()
        c.step()
    torch.cuda.synchronize()
    assert fp8.fp8_get_status() == 0
    keep = [i for i in range(16) if i != 10]  # the gradient's scale itself: written by the separate cast only
    for da, db, dc in zip(a.L, b.L, c.L):  # the in-place step also tracks the master's amax (st[3])
        assert torch.equal(da["sc"], db["sc"]) and torch.equal(da["st"][:3], db["st"][:3]), da["name"]
        assert torch.equal(db["sc"][keep], dc["sc"][keep]) and torch.equal(db["st"], dc["st"]), da["name"]
        # c casts the gradient inside the Adam pass (its gq is never written)
        assert torch.equal(da["gq"], db["gq"]), da["name"]
        for k in ("wq", "y", "dx", "dw"):
            assert torch.equal(da[k], db[k]) and torch.equal(da[k], dc[k]), (da["name"], k)
        for ka, kb in (("m", "m2"), ("v", "v2"), ("wh", "wh2")):
            assert torch.equal(da[ka], db[kb]) and torch.equal(da[ka], dc[kb]), (da["name"], ka)
            assert torch.equal(db[ka], dc[ka]), (da["name"], ka)  # the state after step 2
    del a, b, c
    torch.cuda.empty_cache()


# Which whole chunks the oracle checks after each of the ten steps: every
# tensor kind of the first and of the last layer, and the embedding.
ADAM_7B_CHECKS = {1: ["l0.qkv"], 2: ["l0.out_proj"], 3: ["l0.fc1"], 4: ["l0.fc2"], 5: ["embedding"],
                  6: ["l31.qkv"], 7: ["l31.out_proj"], 8: ["l31.fc1"], 9: ["l31.fc2"],
                  10: ["l0.qkv", "l31.fc2"]}
ADAM_7B_SLICE = 1 << 25  # oracle memory bound: whole chunks are checked in slices of at most this


def _stored_max(t, fmt):
    view = t.view(torch.float8_e4m3fn) if fmt == "e4m3" else t.view(torch.float16)
    return view.float().abs().max().item()


@pytest.mark.parametrize("out_of_place", [False, True])
def test_gpt7b_adam_full_model_ten_steps(out_of_place):
    """The decoupled Adam over all 129 per-tensor chunks of GPT-7B
    (6,648,496,128 parameters, one call per step; in place, and out of place
    as the benchmark runs it, alternating two buffer sets) for ten steps, each step
    with fresh E5M2 gradients ~N(0, 1e-3) x mu for every chunk.  After every
    step the chunks of ADAM_7B_CHECKS are checked whole against the oracle,
    fed the GPU's own state from the step before (scales bit-equal, master
    within 1 FP16 ULP plus the binary32 step term, v within 1 FP16 ULP, m
    within 1 code); and every chunk's three scales are checked against the
    scale rule on its stored values (margin 0: the largest stored magnitude
    is in the format's top binade, [224, 448] for E4M3 and [32752, 65504]
    for FP16, or the tensor is zero with scale 1)."""
    from profile_cases import build_adam_state
    from test_gpu_parity import HP, MAX_TIES, check_adam_chunk, snapshot
    from fp8_mixed_precision_tensor_b200.adam_state import FP8Adam

    specs = synth.gpt7b_adam_chunks()
    assert sum(n for _, n in specs) == 6648496128 and len(specs) == 129
    names = [name for name, _ in specs]
    states = build_adam_state(specs, spare=out_of_place)
    chunks = [st.chunk for st in states]
    opt = FP8Adam(states, margin=0, out_of_place=out_of_place, **HP)
    ties = []
    for step in range(1, 11):
        if step > 1:  # fresh gradients for every chunk
            for ci, (st, (_, n)) in enumerate(zip(states, specs)):
                g = synth.device_normal((n,), 1e-3, synth.key_seed("adam7b", step, ci), torch.float32, "cuda")
                st.set_gradient(g, 2.0 ** 10)
                del g
        picks = [names.index(x) for x in ADAM_7B_CHECKS[step]]
        before = {i: snapshot(chunks[i]) for i in picks}
        opt.step()  # step `step` (out of place: into the other buffer set, which then holds the state)
        assert opt.t == step
        assert fp8.fp8_get_status() == 0, step
        chunks = [st.chunk for st in states]
        for i in picks:
            check_adam_chunk(before[i], chunks[i], step, ties=ties, slices=-(-specs[i][1] // ADAM_7B_SLICE))
        before.clear()
        for name, c in zip(names, chunks):
            for t, sc, fmt, lo, hi in ((c.m, c.m_scale, "e4m3", 224.0, 448.0), (c.v, c.v_scale, "f16", 32752.0, 65504.0),
                                       (c.w, c.w_scale, "f16", 32752.0, 65504.0)):
                top = _stored_max(t, fmt)
                s = sc.item()
                assert np.frexp(s)[0] == 0.5, (step, name, fmt, s)
                assert (lo <= top <= hi) or (top == 0.0 and s == 1.0), (step, name, fmt, top, s)
    assert len(ties) <= MAX_TIES, ties
