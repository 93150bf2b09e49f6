"""Decoupled FP8 Adam state of weight tensors, and the optimizer over them.

"FP8-LM: Training FP8 Large Language Models", 提案手法 O2: per parameter an
FP8 E5M2 gradient, an FP8 E4M3 first moment, an FP16 second moment and an
FP16 master weight, each tensor with its own power-of-two scale.  The
initial state is the master cast from the high-precision weight at the scale
of its amax (fmt_max 65504), and zero moments with scale 1.  Every number is
produced by the library's kernels (amax, fused scale+cast, Adam); this module
only allocates the buffers and orders the calls.
"""
from __future__ import annotations

import torch

from . import fp8


class AdamTensorState:
    """State of one weight tensor of n parameters on the weight's device.

    weight: fp32 / bf16 / fp16 tensor (its values seed the FP16 master).
    track_master_amax: keep the stored master's amax between steps (the
    step's first pass then skips the master).  e4m3_copy: the step also
    writes the E4M3 copy of the new master (the next forward pass's weight
    operand) into `wq`, with its scale and inverse in `wq_scale`, `wq_inv`.
    spare_buffers: a second set of m, v, w buffers for the out-of-place step
    (the step writes them, then `swap` makes them the state)."""

    def __init__(self, weight: torch.Tensor, margin: int = 0, track_master_amax: bool = False,
                 e4m3_copy: bool = False, spare_buffers: bool = False):
        dev = weight.device
        n = weight.numel()
        f32 = dict(dtype=torch.float32, device=dev)
        self.n = n
        # scalars: g_inv, m/v/w scales, tracked amax, E4M3 copy scale and inverse, gradient amax/scale
        self.scalars = torch.zeros(10, **f32)
        s = self.scalars
        s[1:4] = 1.0
        s[4] = -1.0
        self.g = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.m = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.v = torch.zeros(n, dtype=torch.int16, device=dev)
        self.w = torch.empty(n, dtype=torch.int16, device=dev)
        flat = weight.reshape(-1)
        fp8.fp8_amax(flat, s[8:9])
        fp8.fp8_scale_cast(flat, fp8.FP8_F16S, s[8:9], margin, 1.0, s[3:4], s[9:10], self.w)
        self.wq = torch.empty(n, dtype=torch.uint8, device=dev) if e4m3_copy else None
        self.track_master_amax, self.e4m3_copy = track_master_amax, e4m3_copy
        self.spare = ((torch.empty_like(self.m), torch.empty_like(self.v), torch.empty_like(self.w))
                      if spare_buffers else None)
        self._make_chunk()

    def _make_chunk(self) -> None:
        s = self.scalars
        self.chunk = fp8.AdamChunk(self.g, s[0:1], self.m, s[1:2], self.v, s[2:3], self.w, s[3:4],
                                   s[4:5] if self.track_master_amax else None, self.wq,
                                   s[5:6] if self.e4m3_copy else None, s[6:7] if self.e4m3_copy else None)

    def swap(self) -> None:
        """After an out-of-place step: the spare buffers hold the new state."""
        m, v, w = self.spare
        self.spare = (self.m, self.v, self.w)
        self.m, self.v, self.w = m, v, w
        self._make_chunk()

    @property
    def wq_scale(self) -> torch.Tensor:
        return self.scalars[5:6]

    @property
    def wq_inv(self) -> torch.Tensor:
        return self.scalars[6:7]

    def set_gradient(self, grad: torch.Tensor, mu: float, margin: int = 0, grad_amax: torch.Tensor | None = None,
                     stream=None) -> None:
        """Cast a high-precision gradient into the E5M2 buffer ("FP8-LM", 提案手法
        O1: g' = mu g, scale from amax(mu g)); grad_amax, when given, is a device
        scalar already holding amax|grad| (e.g. the wgrad GEMM's fused amax)."""
        s = self.scalars
        flat = grad.reshape(-1)
        if grad_amax is None:
            fp8.fp8_amax(flat, s[7:8], stream=stream)
            grad_amax = s[7:8]
        fp8.fp8_scale_cast(flat, fp8.FP8_E5M2, grad_amax, margin, mu, s[8:9], s[0:1], self.g, stream=stream)


class FP8Adam:
    """One decoupled FP8 Adam step over several tensors' states per call
    (one launch sequence for all of them), with the workspace it needs.
    out_of_place: every state has spare buffers; each step writes the new
    state into them (fp8_adam_step_into: one pass over the state while the
    scales hold) and swaps them in."""

    def __init__(self, states: list[AdamTensorState], lr: float, beta1: float = 0.9, beta2: float = 0.95,
                 eps: float = 1e-8, margin: int = 0, out_of_place: bool = False):
        self.states = states
        self.hp = dict(lr=lr, beta1=beta1, beta2=beta2, eps=eps)
        self.margin = margin
        self.t = 0
        self.out_of_place = out_of_place
        if out_of_place and any(s.spare is None for s in states):
            raise ValueError("the out-of-place step needs states made with spare_buffers=True")
        # the packed chunk and dest arrays of the two buffer assignments (the
        # out-of-place step alternates between them)
        self._packs, self._parity = [None, None], 0
        self._pack()
        dev = states[0].g.device
        self.workspace = torch.zeros(fp8.fp8_adam_workspace_bytes(len(states)) // 4, dtype=torch.float32,
                                     device=dev)

    def _pack(self) -> None:
        k = self._parity
        if self._packs[k] is None:
            self._packs[k] = (fp8.pack_adam_chunks([s.chunk for s in self.states]),
                              fp8.pack_adam_dests([s.spare for s in self.states]) if self.out_of_place else None)
        self.chunks, self.dests = self._packs[k]

    def step(self, stream=None) -> None:
        self.t += 1
        if not self.out_of_place:
            fp8.fp8_adam_step(self.chunks, step=self.t, margin=self.margin, workspace=self.workspace,
                              stream=stream, **self.hp)
            return
        fp8.fp8_adam_step_into(self.chunks, self.dests, step=self.t, margin=self.margin,
                               workspace=self.workspace, stream=stream, **self.hp)
        for s in self.states:
            s.swap()
        self._parity ^= 1
        self._pack()
