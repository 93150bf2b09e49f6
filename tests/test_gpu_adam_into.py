"""The out-of-place Adam step (fp8_adam_step_into) against the in-place step.

Both run the same arithmetic ("FP8-LM: Training FP8 Large Language Models",
提案手法 O2: FP8 gradient and first moment, FP16 second moment and master,
just-in-time per-tensor scales), so the new state must agree bit for bit:
codes, FP16 values, scales, the tracked master amax and the E4M3 copy.  The
out-of-place step predicts that each new scale equals the old one and updates
a chunk a second time when that was wrong; the cases here take both branches
(read back from the workspace's per-chunk flag word, bit 3) and cross the
launch-group boundary of the chunk table.  The in-place step is held to the
oracle by test_gpu_parity.py; one case here also checks the out-of-place
result against the oracle directly.
"""
import numpy as np
import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8, synth

from test_gpu_parity import (F32, HP, MAX_TIES, _stored_amax, _with_tracking, check_adam_chunk, make_adam_state,
                             scalar, snapshot)

pytestmark = pytest.mark.gpu

WS_FLAGS, FLAG_REDO, WS_FLOATS = 10, 8, 16


def _clone(chunks):
    """An independent copy of every buffer and scalar of the chunks."""
    out = []
    for c in chunks:
        kw = {k: (getattr(c, k).clone() if getattr(c, k) is not None else None)
              for k in ("w_amax", "wq", "wq_scale", "wq_inv")}
        out.append(fp8.AdamChunk(c.g, c.g_inv.clone(), c.m.clone(), c.m_scale.clone(), c.v.clone(),
                                 c.v_scale.clone(), c.w.clone(), c.w_scale.clone(), **kw))
    return out


class IntoRunner:
    """Chunks stepped out of place: each step writes the spare buffers, which
    then become the chunk's state (the old ones become the spares)."""

    def __init__(self, chunks):
        self.chunks = chunks
        self.spare = [(torch.empty_like(c.m), torch.empty_like(c.v), torch.empty_like(c.w)) for c in chunks]
        self.ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(chunks)) // 4, **F32)

    def step(self, step, hp=HP, margin=0):
        fp8.fp8_adam_step_into(self.chunks, self.spare, step=step, margin=margin, workspace=self.ws, **hp)
        new = []
        for c, (m, v, w) in zip(self.chunks, self.spare):
            new.append(fp8.AdamChunk(c.g, c.g_inv, m, c.m_scale, v, c.v_scale, w, c.w_scale, c.w_amax, c.wq,
                                     c.wq_scale, c.wq_inv))
        self.spare = [(c.m, c.v, c.w) for c in self.chunks]
        self.chunks = new

    def redone(self):
        """Per chunk: True where the last step updated it a second time."""
        flags = self.ws.view(-1, WS_FLOATS)[:, WS_FLAGS].view(torch.int32).cpu().numpy()
        return (flags & FLAG_REDO) != 0


def assert_same_state(ref, got, where):
    for r, g in zip(ref, got):
        sr, sg = snapshot(r), snapshot(g)
        for k in ("m", "v", "w", "s_m", "s_v", "s_w"):
            assert np.array_equal(np.asarray(sr[k]), np.asarray(sg[k])), (where, k)
        if r.w_amax is not None:
            assert r.w_amax.item() == g.w_amax.item(), where
            if sg["w"].size:
                assert g.w_amax.item() == _stored_amax(sg), where
        if r.wq_scale is not None:
            assert r.wq_scale.item() == g.wq_scale.item() and r.wq_inv.item() == g.wq_inv.item(), where
            assert torch.equal(r.wq, g.wq), where


@pytest.mark.parametrize("track,wq", [(False, False), (True, True), (False, True)])
def test_adam_into_equals_in_place_step(track, wq):
    """Six steps from zero moments, chunks with ragged ends, an empty chunk and
    a chunk of zero gradients (whose scales never change): the out-of-place
    state equals the in-place state after every step; step 1 redoes every
    chunk whose moments change scale, the zero-gradient chunk keeps its
    prediction from step 2 on."""
    sizes = [65536, 4099, 1, 0, 300000, 8192]
    base = make_adam_state(sizes, ("adam-into", track, wq))
    base[5].g.zero_()
    if track or wq:
        base = _with_tracking(base, wq=wq, track=track)
    ref, into = base, IntoRunner(_clone(base))
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(sizes)) // 4, **F32)
    held = 0
    for step in range(1, 7):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        into.step(step)
        assert fp8.fp8_get_status() == 0
        assert_same_state(ref, into.chunks, step)
        r = into.redone()
        if step == 1:
            assert r[0] and r[1] and r[4]
        if step >= 2:
            assert not r[5]
        held += int(np.count_nonzero(~r[[0, 1, 2, 4]]))
    assert held > 0  # some chunks with a moving state also kept their prediction


def test_adam_into_held_predictions_with_unchanged_moments():
    """beta1 = beta2 = 0 and a fixed gradient: from step 2 on the new moments
    equal the old ones, the master moves by ~lr, and every chunk keeps its
    scales (one pass only); the state still equals the in-place step's."""
    hp = dict(HP, beta1=0.0, beta2=0.0, lr=1e-6)
    sizes = [65536 + 7, 4096, 300000]
    base = _with_tracking(make_adam_state(sizes, ("adam-into-held",)), wq=True)
    ref, into = base, IntoRunner(_clone(base))
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(sizes)) // 4, **F32)
    for step in (1, 2, 3):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **hp)
        into.step(step, hp=hp)
        assert fp8.fp8_get_status() == 0
        assert_same_state(ref, into.chunks, step)
        assert into.redone().all() if step == 1 else not into.redone().any(), step


def test_adam_into_many_chunks_two_launch_groups():
    """300 chunks (more than one launch's chunk table): the workspace offsets
    of the second group and its redo pass."""
    sizes = [37 + 16 * i for i in range(300)]
    base = _with_tracking(make_adam_state(sizes, ("adam-into-many",)), wq=True)
    ref, into = base, IntoRunner(_clone(base))
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(sizes)) // 4, **F32)
    for step in (1, 2):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        into.step(step)
        assert fp8.fp8_get_status() == 0
        assert_same_state(ref, into.chunks, step)


def test_adam_into_vs_oracle():
    """Two steps (the second from the GPU's own first-step state), each
    against the oracle."""
    sizes = [65536, 4099, 300000]
    into = IntoRunner(make_adam_state(sizes, ("adam-into-oracle",), steps_done=4))
    ties = []
    for step in (5, 6):
        before = [snapshot(c) for c in into.chunks]
        into.step(step)
        assert fp8.fp8_get_status() == 0
        for b, c in zip(before, into.chunks):
            check_adam_chunk(b, c, step, ties=ties)
    assert len(ties) <= MAX_TIES, ties


def test_adam_into_rejects_bad_destinations():
    chunks = make_adam_state([64], ("adam-into-bad",))
    c = chunks[0]
    ws = torch.zeros(16, **F32)
    with pytest.raises(fp8.FP8Error):  # the new m over the old one
        fp8.fp8_adam_step_into(chunks, [(c.m, torch.empty_like(c.v), torch.empty_like(c.w))], step=1, margin=0,
                               workspace=ws, **HP)
    with pytest.raises(fp8.FP8Error):  # unaligned
        buf = torch.empty(80, dtype=torch.uint8, device="cuda")
        fp8.fp8_adam_step_into(chunks, [(buf[8:72], torch.empty_like(c.v), torch.empty_like(c.w))], step=1,
                               margin=0, workspace=ws, **HP)
    with pytest.raises(ValueError):
        fp8.fp8_adam_step_into(chunks, [], step=1, margin=0, workspace=ws, **HP)
    assert scalar().item() == 0.0  # the device is still usable


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_adam_sharded_into_ranks_equal_whole_tensor_step(world):
    """"FP8-LM", 提案手法 O3 out of place: ranks holding slices of every
    tensor, run one after another on this GPU (stats_into on each, a max over
    their workspaces, apply_into on each, then the buffer sets swap), end
    with exactly the state, scales and E4M3 copy of the whole-tensor in-place
    step, over three steps (step 1 redoes every tensor whose moments change
    scale), through ShardedAdam's two halves (its step puts the collective
    between them)."""
    from fp8_mixed_precision_tensor_b200 import zero
    from test_gpu_parity import _reduce_max_int32

    sizes = [65536 + 5, 4099, 16, 300000]
    ref = _with_tracking(make_adam_state(sizes, ("adam-shard-into",)), wq=True, track=False)
    full = _clone(ref)
    spare = [(torch.empty_like(c.m), torch.empty_like(c.v), torch.empty_like(c.w)) for c in full]
    bounds = [[zero.shard_bounds(n, world, r) for n in sizes] for r in range(world)]
    opts = [zero.ShardedAdam([zero.shard_chunk(c, lo, hi) for c, (lo, hi) in zip(full, bounds[r])],
                             dests=[zero.shard_dest(d, lo, hi) for d, (lo, hi) in zip(spare, bounds[r])])
            for r in range(world)]
    ws_ref = torch.zeros(fp8.fp8_adam_workspace_bytes(len(sizes)) // 4, **F32)
    sets = [[(c.m, c.v, c.w) for c in full], spare]
    for step in (1, 2, 3):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws_ref, **HP)
        for o in opts:
            o.stats(t=step, margin=0, **HP)
        _reduce_max_int32([o.workspace for o in opts])
        for o in opts:
            o.apply(t=step, margin=0, **HP)
        assert fp8.fp8_get_status() == 0
        new = sets[step % 2]  # the whole tensors behind this step's destination slices
        for k, c in enumerate(ref):
            s = snapshot(c)
            m, v, w = new[k]
            assert np.array_equal(m.cpu().numpy(), s["m"]), (step, k)
            assert np.array_equal(v.cpu().numpy().view(np.uint16), s["v"]), (step, k)
            assert np.array_equal(w.cpu().numpy().view(np.uint16), s["w"]), (step, k)
            assert torch.equal(full[k].wq, c.wq)
            for o in opts:
                mine = o.current[k]
                assert (mine.m_scale.item(), mine.v_scale.item(), mine.w_scale.item()) == \
                    (s["s_m"], s["s_v"], s["s_w"]), (step, k)
                assert (mine.wq_scale.item(), mine.wq_inv.item()) == (c.wq_scale.item(), c.wq_inv.item())


@pytest.mark.parametrize("grad_margin,mu", [(0, 2.0 ** 10), (1, 1.0)])
def test_adam_into_castgrad_equals_cast_then_step(grad_margin, mu):
    """The gradient cast in the out-of-place pass (each chunk's g the bf16 dW,
    its amax given): over three steps with fresh gradients, the new state,
    scales, E4M3 copy and the gradient's inverse scale equal those of
    fp8_scale_cast (bf16 dW -> E5M2, mu, margin) followed by the
    out-of-place step on the stored codes, bit for bit -- chunks with ragged
    ends, an empty chunk and a gradient of zeros; step 1 from zero moments
    (every chunk redone)."""
    sizes = [65536, 4099, 1, 0, 300000, 8192]
    base = _with_tracking(make_adam_state(sizes, ("adam-castgrad", grad_margin)), wq=True, track=False)
    ref, fus = IntoRunner(_clone(base)), IntoRunner(_clone(base))
    f32 = dict(dtype=torch.float32, device="cuda")
    for step in (1, 2, 3):
        dws = [synth.device_normal((n,), 1e-3, 77 * step + i, torch.bfloat16, "cuda") for i, n in enumerate(sizes)]
        dws[5].zero_()
        amax = [torch.zeros(1, **f32) for _ in sizes]
        for dw, a in zip(dws, amax):
            fp8.fp8_amax(dw, a)
        # reference: the gradient cast kernel, then the step on the stored codes
        for c, dw, a in zip(ref.chunks, dws, amax):
            s = torch.zeros(1, **f32)
            fp8.fp8_scale_cast(dw, fp8.FP8_E5M2, a, grad_margin, mu, s, c.g_inv, c.g)
        ref.step(step)
        # fused: the same step reading the bf16 gradients
        chunks = [fp8.AdamChunk(dw, c.g_inv, c.m, c.m_scale, c.v, c.v_scale, c.w, c.w_scale, None, c.wq,
                                c.wq_scale, c.wq_inv) for c, dw in zip(fus.chunks, dws)]
        fp8.fp8_adam_step_into_castgrad(chunks, fus.spare, amax, mu, grad_margin, step=step, margin=0,
                                        workspace=fus.ws, **HP)
        fus.chunks = [fp8.AdamChunk(c.g, c.g_inv, m, c.m_scale, v, c.v_scale, w, c.w_scale, None, c.wq, c.wq_scale,
                                    c.wq_inv) for c, (m, v, w) in zip(fus.chunks, fus.spare)]
        fus.spare = [(c.m, c.v, c.w) for c in chunks]
        assert fp8.fp8_get_status() == 0
        assert_same_state(ref.chunks, fus.chunks, step)
        for r, f in zip(ref.chunks, fus.chunks):
            assert r.g_inv.item() == f.g_inv.item(), step
        if step == 1:
            assert fus.redone()[[0, 1, 4]].all()


def test_adam_into_castgrad_rejects_bad_arguments():
    chunks = make_adam_state([64], ("adam-castgrad-bad",))
    c = chunks[0]
    dw = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    ch = [fp8.AdamChunk(dw, c.g_inv, c.m, c.m_scale, c.v, c.v_scale, c.w, c.w_scale)]
    dst = [(torch.empty_like(c.m), torch.empty_like(c.v), torch.empty_like(c.w))]
    ws = torch.zeros(16, **F32)
    a = scalar()
    with pytest.raises(fp8.FP8Error):  # mu not a power of two
        fp8.fp8_adam_step_into_castgrad(ch, dst, [a], 3.0, 0, step=1, margin=0, workspace=ws, **HP)
    with pytest.raises(fp8.FP8Error):  # margin out of range
        fp8.fp8_adam_step_into_castgrad(ch, dst, [a], 1.0, 65, step=1, margin=0, workspace=ws, **HP)
    with pytest.raises(ValueError):
        fp8.fp8_adam_step_into_castgrad(ch, dst, [], 1.0, 0, step=1, margin=0, workspace=ws, **HP)
