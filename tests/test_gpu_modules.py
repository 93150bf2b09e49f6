"""The multi-rank modules on the GPU, one rank: FP8GradAllReduce ("FP8-LM",
提案手法 O1 with Eq. 3) and ShardedAdam (提案手法 O3), first without a
process group, then inside a one-rank NCCL group so that the collective calls
(MAX and SUM all-reduce, all-to-all, all-gather) run on device buffers
exactly as they would with more ranks.  Results against the oracle's FP8
all-reduce and against the plain Adam step."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from fp8_mixed_precision_tensor_b200 import allreduce, fp8, synth, zero
from _util import assert_codes_equal, to_dev
from test_gpu_parity import HP, make_adam_state, snapshot

pytestmark = pytest.mark.gpu


@pytest.fixture
def nccl_one_rank():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        yield
    finally:
        torch.cuda.synchronize()
        dist.destroy_process_group()


def _check_allreduce(scaling):
    n = 300000 + 37
    ar = allreduce.FP8GradAllReduce(n, "cuda", scaling=scaling, theta=0.0, interval=2)
    mu, clean = 1.0, 0
    for step in range(3):
        g = synth.normal_f32((n,), 1e-4, "mod-ar", scaling, step)
        g[:16] = np.float32(0.5)
        out = ar(to_dev(g))
        want = oracle.fp8_allreduce([g], oracle.E5M2, 0, mu)
        assert ar.scalars[1].item() == want["S"]
        assert_codes_equal(out.cpu().numpy(), want["codes"], None, f"{scaling} step {step}")
        assert_codes_equal(ar.all_gather().cpu().numpy(), want["codes"], None, "all_gather")
        assert ar.g_inv.item() == float(np.float32(1.0 / want["S"]))
        if scaling == "auto":
            mu, clean = oracle.mu_update(mu, clean, want["sum_counts"][1], n, 0.0, 2, 2.0 ** -16, 1.0)
        assert ar.mu.item() == mu
    assert fp8.fp8_get_status() == 0


def _check_sharded_adam(out_of_place=False):
    sizes = [65536 + 5, 4099]
    ref = make_adam_state(sizes, ("mod-zero",))
    mine = make_adam_state(sizes, ("mod-zero",))
    dests = ([zero.shard_dest((torch.empty_like(c.m), torch.empty_like(c.v), torch.empty_like(c.w)), 0,
                              c.g.numel()) for c in mine] if out_of_place else None)
    opt = zero.ShardedAdam([zero.shard_chunk(c, 0, c.g.numel()) for c in mine], dests=dests)
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(ref)) // 4, dtype=torch.float32, device="cuda")
    for step in (1, 2, 3):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        opt.step(t=step, margin=0, **HP)
        for r, c in zip(ref, opt.current):
            sr, sc = snapshot(r), snapshot(c)
            for k in ("m", "v", "w"):
                assert np.array_equal(sr[k], sc[k]), (step, k)
            assert (c.m_scale.item(), c.v_scale.item(), c.w_scale.item()) == (sr["s_m"], sr["s_v"], sr["s_w"])
    assert fp8.fp8_get_status() == 0


@pytest.mark.parametrize("scaling", ["auto", "post"])
def test_allreduce_module_without_process_group(scaling):
    _check_allreduce(scaling)


@pytest.mark.parametrize("out_of_place", [False, True])
def test_sharded_adam_module_without_process_group(out_of_place):
    _check_sharded_adam(out_of_place)


def test_modules_inside_a_one_rank_nccl_group(nccl_one_rank):
    _check_allreduce("auto")
    _check_sharded_adam()
    _check_sharded_adam(out_of_place=True)
