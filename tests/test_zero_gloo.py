"""Element-sharded FP8 Adam ("FP8-LM", 提案手法 O3), host side, on CPU:
slice bounds, the MAX reduction of the Adam workspace over gloo ranks, and
ShardedAdam's stats -> reduce -> apply order with the two device halves
replaced by fakes that run the oracle on CPU tensors.  World size 2 (and 3
for the reduction)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from fp8_mixed_precision_tensor_b200 import fp8, synth, zero

HP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8)
WS_FLOATS = 16  # floats of workspace per chunk (fp8_adam_workspace_bytes / 4)


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 4099, 65536, 1000003])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_bounds_partition(n, world):
    bounds = [zero.shard_bounds(n, world, r) for r in range(world)]
    pos = 0
    for lo, hi in bounds:
        assert lo == pos and lo <= hi and (lo == hi or lo % zero.SHARD_ALIGN == 0)
        pos = hi
    assert pos == n
    sizes = [hi - lo for lo, hi in bounds if hi > lo]
    assert all(s == sizes[0] for s in sizes[:-1]) and (not sizes or sizes[-1] <= sizes[0])
    with pytest.raises(ValueError):
        zero.shard_bounds(n, world, world)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)


RANK_WORDS = [
    [0.0, 1.5, float("nan"), 3e-45, float("inf"), 7.0, 0.0],
    [2.0, 1.0, 5.0, 0.0, 1.0, float("nan"), 1e-38],
    [1.0, 1.75, 0.0, 1e-45, 3.0, 2.0, 0.0],
]


def _reduce_worker(rank, world, port):
    _init(rank, world, port)
    try:
        ws = torch.tensor(RANK_WORDS[rank], dtype=torch.float32)
        zero.reduce_workspace(ws)
        cols = np.array(RANK_WORDS[:world], dtype=np.float32)
        for j in range(cols.shape[1]):
            col = cols[:, j]
            expect = np.float32("nan") if np.isnan(col).any() else col.max()
            got = ws[j].item()
            assert (np.isnan(got) and np.isnan(expect)) or got == expect, (j, got, expect)
        assert not torch.signbit(ws).any()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_reduce_workspace_is_an_elementwise_max_with_nan_winning(world):
    mp.spawn(_reduce_worker, args=(world, _free_port()), nprocs=world)


# ---------------------------------------------------------------- ShardedAdam
def _stored_state(n, key):
    gf = synth.normal_f32((n,), 1e-3, "zero", key, "g")
    gf[3] = 0.02
    w = synth.normal_f32((n,), 0.02, "zero", key, "w")
    w[n - 2] = 0.7
    _, sg = oracle.compute_scale(oracle.amax(gf), oracle.E5M2, 0, mu=2.0 ** 10)
    _, s_w = oracle.compute_scale(oracle.amax(w), oracle.F16, 0)
    m0 = synth.normal_f32((n,), 1e-4, "zero", key, "m")
    _, s_m = oracle.compute_scale(oracle.amax(m0), oracle.E4M3, 0)
    v0 = np.abs(synth.normal_f32((n,), 1e-7, "zero", key, "v"))
    _, s_v = oracle.compute_scale(oracle.amax(v0), oracle.F16, 0)
    return (oracle.cast(gf, oracle.E5M2, sg), 1 / sg, oracle.cast(m0, oracle.E4M3, s_m), s_m,
            oracle.cast(v0, oracle.F16, s_v), s_v, oracle.cast(w, oracle.F16, s_w), s_w)


def _to_chunk(st, lo, hi):
    gq, g_inv, mq, s_m, vh, s_v, wh, s_w = st
    f = lambda x: torch.tensor([x], dtype=torch.float32)
    return fp8.AdamChunk(torch.from_numpy(gq[lo:hi].copy()), f(g_inv), torch.from_numpy(mq[lo:hi].copy()),
                         f(s_m), torch.from_numpy(vh[lo:hi].copy().view(np.int16)), f(s_v),
                         torch.from_numpy(wh[lo:hi].copy().view(np.int16)), f(s_w))


def _chunk_args(c):
    return (c.g.numpy(), c.g_inv.item(), c.m.numpy(), c.m_scale.item(), c.v.numpy().view(np.uint16),
            c.v_scale.item(), c.w.numpy().view(np.uint16), c.w_scale.item())


def _fake_stats(chunks, lr, beta1, beta2, eps, t, margin, ws, stream=None):
    ws.zero_()
    for i, c in enumerate(chunks):
        out = oracle.adam_step(*_chunk_args(c), lr, beta1, beta2, eps, t, margin)
        ws[i * WS_FLOATS:i * WS_FLOATS + 3] = torch.tensor(out["amax"], dtype=torch.float32)


def _fake_apply(chunks, lr, beta1, beta2, eps, t, margin, ws, stream=None):
    for i, c in enumerate(chunks):
        amax = tuple(float(x) for x in ws[i * WS_FLOATS:i * WS_FLOATS + 3])
        out = oracle.adam_step(*_chunk_args(c), lr, beta1, beta2, eps, t, margin, amax_in=amax)
        c.m.copy_(torch.from_numpy(out["mq"]))
        c.v.copy_(torch.from_numpy(out["vh"].view(np.int16)))
        c.w.copy_(torch.from_numpy(out["wh"].view(np.int16)))
        c.m_scale.fill_(out["s_m"])
        c.v_scale.fill_(out["s_v"])
        c.w_scale.fill_(out["s_w"])


SIZES = (4099, 1040)


def _sharded_worker(rank, world, port):
    _init(rank, world, port)
    try:
        fp8.pack_adam_chunks = lambda chunks: chunks
        fp8.fp8_adam_workspace_bytes = lambda n: 4 * WS_FLOATS * n
        fp8.fp8_adam_stats = _fake_stats
        fp8.fp8_adam_apply = _fake_apply
        states = [_stored_state(n, str(n)) for n in SIZES]
        bounds = [zero.shard_bounds(n, world, rank) for n in SIZES]
        mine = [_to_chunk(st, lo, hi) for st, (lo, hi) in zip(states, bounds)]
        opt = zero.ShardedAdam(mine)
        whole = [list(st) for st in states]
        for t in (1, 2):
            opt.step(t=t, margin=0, **HP)
            for k, st in enumerate(whole):
                out = oracle.adam_step(*st, t=t, margin=0, **HP)
                st[2], st[3], st[4], st[5], st[6], st[7] = (out["mq"], out["s_m"], out["vh"], out["s_v"],
                                                            out["wh"], out["s_w"])
                lo, hi = bounds[k]
                c = mine[k]
                assert (c.m_scale.item(), c.v_scale.item(), c.w_scale.item()) == (out["s_m"], out["s_v"],
                                                                                   out["s_w"])
                assert np.array_equal(c.m.numpy(), out["mq"][lo:hi])
                assert np.array_equal(c.v.numpy().view(np.uint16), out["vh"][lo:hi])
                assert np.array_equal(c.w.numpy().view(np.uint16), out["wh"][lo:hi])
    finally:
        dist.destroy_process_group()


def test_sharded_adam_over_gloo_equals_the_whole_tensor_step():
    mp.spawn(_sharded_worker, args=(2, _free_port()), nprocs=2)


def _fake_stats_into(chunks, dests, lr, beta1, beta2, eps, t, margin, ws, stream=None):
    _fake_stats(chunks, lr, beta1, beta2, eps, t, margin, ws)
    for m, v, w in dests:  # the predicted-scale state: overwritten by the apply half here
        m.fill_(0x55), v.fill_(0x55), w.fill_(0x55)


def _fake_apply_into(chunks, dests, lr, beta1, beta2, eps, t, margin, ws, stream=None):
    for i, (c, (m, v, w)) in enumerate(zip(chunks, dests)):
        amax = tuple(float(x) for x in ws[i * WS_FLOATS:i * WS_FLOATS + 3])
        out = oracle.adam_step(*_chunk_args(c), lr, beta1, beta2, eps, t, margin, amax_in=amax)
        m.copy_(torch.from_numpy(out["mq"]))
        v.copy_(torch.from_numpy(out["vh"].view(np.int16)))
        w.copy_(torch.from_numpy(out["wh"].view(np.int16)))
        c.m_scale.fill_(out["s_m"])
        c.v_scale.fill_(out["s_v"])
        c.w_scale.fill_(out["s_w"])


def _sharded_into_worker(rank, world, port):
    """The out-of-place halves: stats_into -> MAX reduce -> apply_into, then
    the new buffers become the state and the old ones the next step's
    destination (the inputs of a step are never its outputs)."""
    _init(rank, world, port)
    try:
        fp8.pack_adam_chunks = lambda chunks: chunks
        fp8.pack_adam_dests = lambda dests: dests
        fp8.fp8_adam_workspace_bytes = lambda n: 4 * WS_FLOATS * n
        fp8.fp8_adam_stats_into = _fake_stats_into
        fp8.fp8_adam_apply_into = _fake_apply_into
        states = [_stored_state(n, str(n)) for n in SIZES]
        bounds = [zero.shard_bounds(n, world, rank) for n in SIZES]
        mine = [_to_chunk(st, lo, hi) for st, (lo, hi) in zip(states, bounds)]
        spare = [zero.shard_dest((torch.empty(n, dtype=torch.uint8), torch.empty(n, dtype=torch.int16),
                                  torch.empty(n, dtype=torch.int16)), lo, hi)
                 for n, (lo, hi) in zip(SIZES, bounds)]
        opt = zero.ShardedAdam(mine, dests=spare)
        whole = [list(st) for st in states]
        for t in (1, 2, 3):
            before = [(c.m, c.v, c.w) for c in opt.current]
            opt.step(t=t, margin=0, **HP)
            for k, st in enumerate(whole):
                out = oracle.adam_step(*st, t=t, margin=0, **HP)
                st[2], st[3], st[4], st[5], st[6], st[7] = (out["mq"], out["s_m"], out["vh"], out["s_v"],
                                                            out["wh"], out["s_w"])
                lo, hi = bounds[k]
                c = opt.current[k]
                assert all(a is not b for a, b in zip((c.m, c.v, c.w), before[k]))
                assert all(a is b for a, b in zip(opt.spare[k], before[k]))
                assert (c.m_scale.item(), c.v_scale.item(), c.w_scale.item()) == (out["s_m"], out["s_v"],
                                                                                   out["s_w"])
                assert np.array_equal(c.m.numpy(), out["mq"][lo:hi])
                assert np.array_equal(c.v.numpy().view(np.uint16), out["vh"][lo:hi])
                assert np.array_equal(c.w.numpy().view(np.uint16), out["wh"][lo:hi])
    finally:
        dist.destroy_process_group()


def test_sharded_adam_out_of_place_over_gloo_equals_the_whole_tensor_step():
    mp.spawn(_sharded_into_worker, args=(2, _free_port()), nprocs=2)


def test_shard_dest_checks_its_slice():
    bufs = (torch.empty(100, dtype=torch.uint8), torch.empty(100, dtype=torch.int16),
            torch.empty(100, dtype=torch.int16))
    assert [t.numel() for t in zero.shard_dest(bufs, 16, 48)] == [32, 32, 32]
    with pytest.raises(ValueError):
        zero.shard_dest(bufs, 8, 48)
    with pytest.raises(ValueError):
        zero.shard_dest(bufs, 96, 112)


def test_sharded_adam_rejects_tracked_master_amax():
    st = _stored_state(64, "trk")
    c = _to_chunk(st, 0, 64)
    c.w_amax = torch.tensor([-1.0])
    with pytest.raises(ValueError):
        zero.shard_chunk(c, 0, 32)
    with pytest.raises(ValueError):
        zero.ShardedAdam([c])
