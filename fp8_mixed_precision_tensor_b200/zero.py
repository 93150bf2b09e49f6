"""Element-sharded decoupled FP8 Adam across data-parallel ranks.

"FP8-LM: Training FP8 Large Language Models", 提案手法 O3: the FP8 optimizer
state is partitioned over the ranks ZeRO-style.  Every rank owns one
contiguous slice of every tensor and runs the decoupled Adam step
(提案手法 O2) on its slices only.  The one coupling between ranks is the
per-tensor scale of m, v and w, which comes from the amax of the whole new
tensor: three scalars per tensor, combined by a single MAX all-reduce
between the two halves of the step (fp8_adam_stats, fp8_adam_apply; out of
place, fp8_adam_stats_into and fp8_adam_apply_into, which read the state
once while the scales hold).

Slice boundaries sit on multiples of 16 elements, so every slice of the
1- and 2-byte state arrays starts 16-byte aligned as the kernels require.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import fp8

SHARD_ALIGN = 16


def shard_bounds(n: int, world: int, rank: int, align: int = SHARD_ALIGN) -> tuple[int, int]:
    """[lo, hi) of rank's slice of an n-element tensor: equal runs of whole
    `align`-element groups, the ragged remainder on the last non-empty slice;
    trailing ranks may get an empty slice (lo == hi == n)."""
    if world < 1 or not 0 <= rank < world or n < 0 or align < 1:
        raise ValueError(f"bad shard request n={n} world={world} rank={rank} align={align}")
    groups = -(-n // align)
    per = -(-groups // world)
    lo = min(n, rank * per * align)
    hi = min(n, (rank + 1) * per * align)
    return lo, hi


def reduce_workspace(workspace: torch.Tensor, group=None) -> None:
    """Element-wise MAX of an Adam workspace over the ranks of `group`, in
    place.  Every word is the bit pattern of a float >= 0 (or +NaN), so the
    words are reduced as int32: integer order is the amax order and a NaN
    wins, independent of how the backend treats NaN in a float max."""
    if workspace.dtype != torch.float32:
        raise TypeError("the Adam workspace is float32")
    dist.all_reduce(workspace.view(torch.int32), op=dist.ReduceOp.MAX, group=group)


def shard_chunk(c: fp8.AdamChunk, lo: int, hi: int) -> fp8.AdamChunk:
    """This rank's slice [lo, hi) of one tensor's stored state: views of the
    element arrays and private copies of the scale scalars (every rank keeps
    its own replica of a tensor's scales and rewrites it each step)."""
    if (hi > lo and lo % SHARD_ALIGN) or not 0 <= lo <= hi <= c.g.numel():
        raise ValueError(f"bad slice [{lo}, {hi}) of {c.g.numel()} elements")
    if c.w_amax is not None:
        raise ValueError("tracked master amax is not available in the sharded step")
    view = lambda t: t.reshape(-1)[lo:hi]
    own = lambda t: None if t is None else t.clone()
    return fp8.AdamChunk(view(c.g), own(c.g_inv), view(c.m), own(c.m_scale), view(c.v), own(c.v_scale),
                         view(c.w), own(c.w_scale), None,
                         None if c.wq is None else view(c.wq), own(c.wq_scale), own(c.wq_inv))


def shard_dest(bufs, lo: int, hi: int) -> tuple:
    """This rank's slice [lo, hi) of a tensor's second set of state buffers
    (m, v, w), for the out-of-place step."""
    if (hi > lo and lo % SHARD_ALIGN) or not 0 <= lo <= hi <= bufs[0].numel():
        raise ValueError(f"bad slice [{lo}, {hi}) of {bufs[0].numel()} elements")
    return tuple(t.reshape(-1)[lo:hi] for t in bufs)


class ShardedAdam:
    """The decoupled FP8 Adam step over this rank's slices.  `chunks` holds
    slice i of tensor i on every rank, in the same order; `group` is the
    data-parallel process group (None: the default group).  With `dests`
    (per chunk the matching slices (m, v, w) of a second set of buffers) the
    step is out of place: each step writes the new state into the other set
    and `current` follows it."""

    def __init__(self, chunks: list[fp8.AdamChunk], group=None, dests: list[tuple] | None = None):
        if any(c.w_amax is not None for c in chunks):
            raise ValueError("tracked master amax is not available in the sharded step")
        if dests is not None and len(dests) != len(chunks):
            raise ValueError("one dest per chunk")
        self.current = list(chunks)
        self.spare = None if dests is None else [tuple(d) for d in dests]
        self._packs, self._parity = [None, None], 0
        self._pack()
        self.group = group
        device = chunks[0].g_inv.device
        self.workspace = torch.zeros(fp8.fp8_adam_workspace_bytes(len(chunks)) // 4, dtype=torch.float32,
                                     device=device)

    def _pack(self) -> None:
        k = self._parity
        if self._packs[k] is None:
            self._packs[k] = (fp8.pack_adam_chunks(self.current),
                              None if self.spare is None else fp8.pack_adam_dests(self.spare))
        self.chunks, self.dests = self._packs[k]

    def _reduce(self, stream) -> None:
        if dist.is_available() and dist.is_initialized():  # a group of one rank too
            if stream is None:
                reduce_workspace(self.workspace, self.group)
            else:
                with torch.cuda.stream(stream):
                    reduce_workspace(self.workspace, self.group)

    def stats(self, lr: float, beta1: float, beta2: float, eps: float, t: int, margin: int = 0,
              stream=None) -> None:
        """First half of the step on this rank's slices: the workspace then
        holds their exact new amaxes (out of place, the new slices are also
        written with the predicted scales)."""
        args = (lr, beta1, beta2, eps, t, margin, self.workspace)
        if self.spare is None:
            fp8.fp8_adam_stats(self.chunks, *args, stream=stream)
        else:
            fp8.fp8_adam_stats_into(self.chunks, self.dests, *args, stream=stream)

    def apply(self, lr: float, beta1: float, beta2: float, eps: float, t: int, margin: int = 0,
              stream=None) -> None:
        """Second half, after the workspace was MAX-reduced over the ranks:
        the new scales and the new slices (out of place, the buffer sets then
        swap: `current` holds the new state)."""
        args = (lr, beta1, beta2, eps, t, margin, self.workspace)
        if self.spare is None:
            fp8.fp8_adam_apply(self.chunks, *args, stream=stream)
            return
        fp8.fp8_adam_apply_into(self.chunks, self.dests, *args, stream=stream)
        new = [fp8.AdamChunk(c.g, c.g_inv, m, c.m_scale, v, c.v_scale, w, c.w_scale, None, c.wq, c.wq_scale,
                             c.wq_inv) for c, (m, v, w) in zip(self.current, self.spare)]
        self.spare = [(c.m, c.v, c.w) for c in self.current]
        self.current = new
        self._parity ^= 1
        self._pack()

    def step(self, lr: float, beta1: float, beta2: float, eps: float, t: int, margin: int = 0,
             stream=None) -> None:
        """stats -> MAX all-reduce of the workspace -> apply, all on `stream`
        (a torch.cuda.Stream; the current stream by default), which the
        collective also uses."""
        self.stats(lr, beta1, beta2, eps, t, margin, stream)
        self._reduce(stream)
        self.apply(lr, beta1, beta2, eps, t, margin, stream)
