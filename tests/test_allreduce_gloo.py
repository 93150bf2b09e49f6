"""FP8 gradient all-reduce ("FP8-LM", 提案手法 O1 with Eq. 3, and the
pre-/post-scaling comparison of アブレーション研究), host side, on CPU over
gloo ranks: the shared amax, the all-to-all slice layout, the count
reduction and the order of the mu updates, with the four device kernels
replaced by fakes that run the oracle on CPU tensors.  Each rank's result is
compared with the oracle's all-reduce over every rank's gradient."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from fp8_mixed_precision_tensor_b200 import allreduce, fp8, synth, zero

FMT = {fp8.FP8_E4M3: oracle.E4M3, fp8.FP8_E5M2: oracle.E5M2}


def _fake_amax(x, out, stream=None):
    out.fill_(oracle.amax(x.numpy()))


def _fake_grad_cast(g, fmt, amax, margin, mu, scale_out, inv_out, q, counts=None, stream=None):
    _, S = oracle.grad_scale(amax.item(), FMT[fmt], margin, mu.item())
    codes, c = oracle.cast_counts(g.numpy(), FMT[fmt], S)
    q[:g.numel()] = torch.from_numpy(codes)
    scale_out.fill_(S)
    inv_out.fill_(1.0 / S)
    if counts is not None:
        counts += torch.tensor(c, dtype=torch.int64)


def _fake_sum_codes(rows, n, fmt, out, inv_scale=None, g_inv_out=None, counts=None, stream=None):
    codes, c = oracle.sum_codes(rows[:, :n].numpy(), FMT[fmt])
    out[:n] = torch.from_numpy(codes)
    if g_inv_out is not None:
        g_inv_out.fill_(float(np.float32(inv_scale.item()) * np.float32(1.0 / rows.shape[0])))
    if counts is not None:
        counts += torch.tensor(c, dtype=torch.int64)


def _fake_mu_update(mu, clean, counts, n, theta, interval, mu_min, mu_max, stream=None):
    m, c = oracle.mu_update(mu.item(), int(clean.item()), int(counts[1].item()), n,
                            float(np.float32(theta)), interval, mu_min, mu_max)
    mu.fill_(m)
    clean.fill_(c)
    counts.zero_()


def _patch():
    fp8.fp8_amax = _fake_amax
    fp8.fp8_grad_cast = _fake_grad_cast
    fp8.fp8_sum_codes = _fake_sum_codes
    fp8.fp8_mu_update = _fake_mu_update


def _grads(world, n, step):
    """Every rank's gradient at a step; elements 0..3 agree in sign on all
    ranks (their sum overflows at mu = 1), the rest is small noise."""
    out = []
    for r in range(world):
        g = synth.normal_f32((n,), 1e-4, "ar", world, n, step, r)
        g[:4] = np.float32(1.0 + 0.1 * r)
        g[5] = np.float32(2.0 ** -40)  # underflows once divided by the rank count
        out.append(g)
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, scaling, n):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        _patch()
        ar = allreduce.FP8GradAllReduce(n, "cpu", fmt=fp8.FP8_E5M2, scaling=scaling, theta=0.0, interval=2)
        lo, hi = zero.shard_bounds(n, world, rank)
        mu = {"auto": 1.0, "post": 1.0, "pre": 2.0 ** -int(np.ceil(np.log2(world)))}[scaling]
        clean = 0
        auto_sums = np.zeros(2, dtype=np.int64)
        for step in range(4):
            grads = _grads(world, n, step)
            want = oracle.fp8_allreduce(grads, oracle.E5M2, 0, mu)
            mine = ar(torch.from_numpy(grads[rank]))
            assert ar.scalars[1].item() == want["S"]
            assert np.array_equal(mine.numpy(), want["codes"][lo:hi])
            assert np.array_equal(ar.all_gather().numpy(), want["codes"])
            assert ar.g_inv.item() == float(np.float32(1.0 / want["S"]) * np.float32(1.0 / world))
            if scaling == "auto":
                auto_sums += np.asarray(want["sum_counts"], dtype=np.int64)
                mu, clean = oracle.mu_update(mu, clean, want["sum_counts"][1], n, 0.0, 2, 2.0 ** -16, 1.0)
            assert ar.mu.item() == mu, (step, ar.mu.item(), mu)
        if scaling == "auto":
            # the running totals of the rank-summed counts, not re-summed over the ranks
            r = ar.rates()
            assert (r["sum_underflow"], r["sum_overflow"]) == tuple(auto_sums.tolist()), (r, auto_sums)
            assert auto_sums[1] > 0  # the first step, at mu = 1, saturates elements 0..3
        if scaling == "post":
            assert ar.rates()["sum_overflow"] == 4 * 4  # four steps, elements 0..3 saturate
        if scaling == "pre" and world > 1:
            assert ar.rates()["cast_underflow"] >= 4 * world  # element 5 on every rank, every step
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("scaling", ["auto", "post", "pre"])
def test_fp8_allreduce_over_gloo_matches_the_oracle(world, scaling):
    mp.spawn(_worker, args=(world, _free_port(), scaling, 1000 + 37), nprocs=world)


def test_single_rank_allreduce_is_the_rank_own_requantised_gradient():
    _saved = (fp8.fp8_amax, fp8.fp8_grad_cast, fp8.fp8_sum_codes, fp8.fp8_mu_update)
    try:
        _patch()
        g = _grads(1, 517, 0)[0]
        ar = allreduce.FP8GradAllReduce(517, "cpu", scaling="post")
        out = ar(torch.from_numpy(g))
        want = oracle.fp8_allreduce([g], oracle.E5M2, 0, 1.0)
        assert np.array_equal(out.numpy(), want["codes"])
        assert out.numel() == 517 and ar.all_gather().numel() == 517
    finally:
        fp8.fp8_amax, fp8.fp8_grad_cast, fp8.fp8_sum_codes, fp8.fp8_mu_update = _saved


def test_bad_scaling_name_and_size():
    with pytest.raises(ValueError):
        allreduce.FP8GradAllReduce(16, "cpu", scaling="sideways")
    ar = allreduce.FP8GradAllReduce(16, "cpu")
    with pytest.raises(ValueError):
        ar(torch.zeros(17))
