"""Host logic of the per-tensor Adam state and optimizer (adam_state.py) on
CPU: FP8Adam's out-of-place mode hands each step the current buffers as the
input and the spare set as the destination, swaps the two sets after the
step, and keeps its packed arrays in step with the swap; the in-place mode
updates the same buffers.  The library calls are replaced by fakes that run
the oracle on CPU tensors ("FP8-LM: Training FP8 Large Language Models",
提案手法 O2: the decoupled Adam step on FP8/FP16 state), so the trajectory
must be the oracle's own three-step trajectory whichever mode runs it.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_mixed_precision_tensor_b200 import adam_state, fp8, synth

HP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8)


def _fake_amax(x, out, stream=None):
    out.fill_(float(np.max(np.abs(x.float().numpy()))) if x.numel() else 0.0)


def _fake_scale_cast(x, fmt, amax, margin, mu, scale, inv, q, stream=None):
    ofmt = {fp8.FP8_E4M3: oracle.E4M3, fp8.FP8_E5M2: oracle.E5M2, fp8.FP8_F16S: oracle.F16}[fmt]
    _, s = oracle.compute_scale(amax.item(), ofmt, margin, mu)
    scale.fill_(s)
    inv.fill_(1.0 / s)
    codes = oracle.cast(x.float().numpy().astype(np.float32), ofmt, s)
    q.copy_(torch.from_numpy(codes.view(np.int16) if ofmt == oracle.F16 else codes))


def _oracle_into(c, m_out, v_out, w_out, t):
    out = oracle.adam_step(c.g.numpy(), c.g_inv.item(), c.m.numpy(), c.m_scale.item(),
                           c.v.numpy().view(np.uint16), c.v_scale.item(), c.w.numpy().view(np.uint16),
                           c.w_scale.item(), t=t, margin=0, **HP)
    m_out.copy_(torch.from_numpy(out["mq"]))
    v_out.copy_(torch.from_numpy(out["vh"].view(np.int16)))
    w_out.copy_(torch.from_numpy(out["wh"].view(np.int16)))
    c.m_scale.fill_(out["s_m"])
    c.v_scale.fill_(out["s_v"])
    c.w_scale.fill_(out["s_w"])


def _fake_step(chunks, lr, beta1, beta2, eps, step, margin, workspace, stream=None):
    for c in chunks:
        _oracle_into(c, c.m, c.v, c.w, step)


def _fake_step_into(chunks, dests, lr, beta1, beta2, eps, step, margin, workspace, stream=None):
    for c, (m, v, w) in zip(chunks, dests):
        assert all(a.data_ptr() != b.data_ptr() for a, b in zip((m, v, w), (c.m, c.v, c.w)))
        _oracle_into(c, m, v, w, step)


@pytest.fixture
def fake_library(monkeypatch):
    monkeypatch.setattr(fp8, "fp8_amax", _fake_amax)
    monkeypatch.setattr(fp8, "fp8_scale_cast", _fake_scale_cast)
    monkeypatch.setattr(fp8, "fp8_adam_workspace_bytes", lambda n: 64 * n)
    monkeypatch.setattr(fp8, "pack_adam_chunks", lambda chunks: list(chunks))
    monkeypatch.setattr(fp8, "pack_adam_dests", lambda dests: list(dests))
    monkeypatch.setattr(fp8, "fp8_adam_step", _fake_step)
    monkeypatch.setattr(fp8, "fp8_adam_step_into", _fake_step_into)
    monkeypatch.setattr(fp8, "_ptr", lambda t: None if t is None else t.data_ptr())


def _states(spare, sizes=(4099, 1040)):
    out = []
    for k, n in enumerate(sizes):
        w = torch.from_numpy(synth.normal_f32((n,), 0.02, "host-adam", k, "w"))
        st = adam_state.AdamTensorState(w, spare_buffers=spare)
        g = torch.from_numpy(synth.normal_f32((n,), 1e-3, "host-adam", k, "g"))
        st.set_gradient(g, 2.0 ** 10)
        out.append(st)
    return out


@pytest.mark.parametrize("out_of_place", [False, True])
def test_fp8adam_follows_the_oracle_trajectory(fake_library, out_of_place):
    states = _states(out_of_place)
    ref = [[st.g.numpy().copy(), st.scalars[0].item(), st.m.numpy().copy(), st.scalars[1].item(),
            st.v.numpy().view(np.uint16).copy(), st.scalars[2].item(), st.w.numpy().view(np.uint16).copy(),
            st.scalars[3].item()] for st in states]
    opt = adam_state.FP8Adam(states, out_of_place=out_of_place, **HP)
    first = [(st.m, st.v, st.w) for st in states]
    for t in (1, 2, 3):
        held = [(st.m, st.v, st.w) for st in states]
        opt.step()
        for st, r, h in zip(states, ref, held):
            out = oracle.adam_step(*r, t=t, margin=0, **HP)
            r[2], r[3], r[4], r[5], r[6], r[7] = out["mq"], out["s_m"], out["vh"], out["s_v"], out["wh"], out["s_w"]
            assert np.array_equal(st.m.numpy(), out["mq"]) and st.scalars[1].item() == out["s_m"]
            assert np.array_equal(st.v.numpy().view(np.uint16), out["vh"]) and st.scalars[2].item() == out["s_v"]
            assert np.array_equal(st.w.numpy().view(np.uint16), out["wh"]) and st.scalars[3].item() == out["s_w"]
            moved = st.m is not h[0]
            assert moved == out_of_place  # out of place: the new state sits in the other buffer set
            if out_of_place:
                assert st.spare[0] is h[0] and st.chunk.m is st.m
        # the packed arrays follow the buffers
        assert all(c.m is st.m for c, st in zip(opt.chunks, states))
    if out_of_place:  # after three steps the state is in the second set, the first set is spare
        assert all(st.spare[0] is f[0] for st, f in zip(states, first))


def test_fp8adam_out_of_place_needs_spare_buffers(fake_library):
    with pytest.raises(ValueError):
        adam_state.FP8Adam(_states(False), out_of_place=True, **HP)
