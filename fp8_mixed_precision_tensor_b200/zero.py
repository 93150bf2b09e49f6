"""Element-sharded decoupled FP8 Adam across data-parallel ranks.

"FP8-LM: Training FP8 Large Language Models", 提案手法 O3: the FP8 optimizer
state is partitioned over the ranks ZeRO-style.  Every rank owns one
contiguous slice of every tensor and runs the decoupled Adam step
(提案手法 O2) on its slices only.  The one coupling between ranks is the
per-tensor scale of m, v and w, which comes from the amax of the whole new
tensor: three scalars per tensor, combined by a single MAX all-reduce
between the two halves of the step (fp8_adam_stats, fp8_adam_apply).

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


class ShardedAdam:
    """The decoupled FP8 Adam step over this rank's slices.  `chunks` holds
    slice i of tensor i on every rank, in the same order; `group` is the
    data-parallel process group (None: the default group)."""

    def __init__(self, chunks: list[fp8.AdamChunk], group=None):
        if any(c.w_amax is not None for c in chunks):
            raise ValueError("tracked master amax is not available in the sharded step")
        self.chunks = fp8.pack_adam_chunks(chunks)
        self._keep = chunks
        self.group = group
        device = chunks[0].g_inv.device
        self.workspace = torch.zeros(fp8.fp8_adam_workspace_bytes(len(chunks)) // 4, dtype=torch.float32,
                                     device=device)

    def step(self, lr: float, beta1: float, beta2: float, eps: float, t: int, margin: int = 0,
             stream=None) -> None:
        """stats -> MAX all-reduce of the workspace -> apply, all on `stream`
        (a torch.cuda.Stream; the current stream by default), which the
        collective also uses."""
        args = (lr, beta1, beta2, eps, t, margin, self.workspace)
        fp8.fp8_adam_stats(self.chunks, *args, stream=stream)
        if dist.is_available() and dist.is_initialized():  # a group of one rank too
            if stream is None:
                reduce_workspace(self.workspace, self.group)
            else:
                with torch.cuda.stream(stream):
                    reduce_workspace(self.workspace, self.group)
        fp8.fp8_adam_apply(self.chunks, *args, stream=stream)
