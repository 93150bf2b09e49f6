"""FP8 gradient all-reduce across data-parallel ranks, with auto-scaling.

"FP8-LM: Training FP8 Large Language Models", 提案手法 O1: weight gradients
are communicated in FP8, auto-scaled by mu (g' = mu * g, Eq. 3) so that the
sum over ranks neither overflows nor underflows; アブレーション研究: this
beats dividing by the rank count before the cast (pre-scaling: underflow) or
after the sum (post-scaling: overflow).

One tensor's all-reduce, per rank (every numeric step is a libfp8 kernel;
this module only orders them around the collectives):

  1. amax of the rank's gradient (given, e.g. a wgrad GEMM's output amax,
     or fp8_amax), then a MAX all-reduce of it: the shared amax;
  2. fp8_grad_cast: the rank's payload codes at the shared scale
     S = mu * 2^(floor(log2(fmt_max / amax)) - margin);
  3. an all-to-all: rank j receives every rank's codes of its slice j
     (slices as zero.shard_bounds, so the result feeds zero.ShardedAdam);
  4. fp8_sum_codes: the exact sum of the received codes re-encoded at S,
     and g_inv = 1 / (S * world), the descale of the mean gradient;
  5. with auto-scaling, a SUM all-reduce of the overflow counts and
     fp8_mu_update, which keeps mu on the device and identical on all ranks.

`all_gather()` assembles the whole reduced gradient for a replicated
optimizer.  FP8 codes cross the links: 1 byte per element each way.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import fp8
from .zero import SHARD_ALIGN, shard_bounds

SCALINGS = ("auto", "pre", "post")


def _group_info(group):
    """(world, rank, collectives): collectives run whenever a process group
    exists, a group of one rank included (so its code path is the same)."""
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group), True
    return 1, 0, False


class FP8GradAllReduce:
    """The FP8 all-reduce of one gradient tensor of n elements.

    scaling: "auto" (mu from the rule, starting at mu_init), "post" (mu = 1),
    "pre" (mu = 2^-ceil(log2 world), the power of two at or below 1/world so
    that every scale stays a power of two).  The rule: more than
    theta * n overflows in a step halve mu (not below mu_min); `interval`
    clean steps in a row double it (not above mu_max)."""

    def __init__(self, n: int, device, fmt: int = fp8.FP8_E5M2, margin: int = 0, scaling: str = "auto",
                 group=None, mu_init: float = 1.0, theta: float = 1e-5, interval: int = 100,
                 mu_min: float = 2.0 ** -16, mu_max: float = 1.0):
        if scaling not in SCALINGS:
            raise ValueError(f"scaling must be one of {SCALINGS}")
        self.n, self.fmt, self.margin, self.scaling, self.group = n, fmt, margin, scaling, group
        self.world, self.rank, self.collectives = _group_info(group)
        self.lo, self.hi = shard_bounds(n, self.world, self.rank)
        groups = -(-n // SHARD_ALIGN)
        self.L = -(-groups // self.world) * SHARD_ALIGN  # slice stride (the last slice may be shorter)
        self.rule = dict(theta=theta, interval=interval, mu_min=mu_min, mu_max=mu_max)
        mu = {"auto": mu_init, "post": 1.0, "pre": 2.0 ** -math.ceil(math.log2(self.world))}[scaling]
        f32 = dict(dtype=torch.float32, device=device)
        self.mu = torch.full((1,), mu, **f32)
        self.clean = torch.zeros(1, dtype=torch.int32, device=device)
        self.scalars = torch.zeros(4, **f32)  # shared amax, S, 1/S, g_inv
        self.cast_counts = torch.zeros(2, dtype=torch.int64, device=device)
        self.sum_counts = torch.zeros(2, dtype=torch.int64, device=device)
        # "auto": running total of the summed counts over the ranks (fp8_mu_update
        # clears sum_counts every step once it has read them)
        self.sum_total = torch.zeros(2, dtype=torch.int64, device=device)
        self.send = torch.zeros(self.world * self.L, dtype=torch.uint8, device=device)  # tail stays 0
        self.recv = torch.zeros(self.world, self.L, dtype=torch.uint8, device=device)
        self.out = torch.zeros(self.L, dtype=torch.uint8, device=device)

    @property
    def amax(self):
        return self.scalars[0:1]

    @property
    def g_inv(self):
        """Descale of the rank's slice of the mean gradient: 1 / (S * world)."""
        return self.scalars[3:4]

    def __call__(self, g: torch.Tensor, g_amax: torch.Tensor | None = None) -> torch.Tensor:
        """Reduce `g` (n elements, f32/bf16/f16, device).  g_amax: the rank's
        own amax of g (device float), computed here when None.  Returns this
        rank's slice [lo, hi) of the summed gradient as codes at scale S;
        their mean-gradient descale is `g_inv`."""
        if g.numel() != self.n:
            raise ValueError(f"expected {self.n} elements, got {g.numel()}")
        if g_amax is None:
            fp8.fp8_amax(g, self.amax)
        else:
            self.amax.copy_(g_amax.reshape(1))
        if self.collectives:
            # amaxes are floats >= 0 (or +NaN): their bit patterns order as int32
            dist.all_reduce(self.amax.view(torch.int32), op=dist.ReduceOp.MAX, group=self.group)
        fp8.fp8_grad_cast(g, self.fmt, self.amax, self.margin, self.mu, self.scalars[1:2], self.scalars[2:3],
                          self.send, self.cast_counts)
        if self.collectives:
            dist.all_to_all_single(self.recv.view(-1), self.send, group=self.group)
            rows = self.recv
        else:
            rows = self.send.view(1, -1)
        fp8.fp8_sum_codes(rows, self.hi - self.lo, self.fmt, self.out, self.scalars[2:3], self.g_inv,
                          self.sum_counts)
        if self.scaling == "auto":
            if self.collectives:
                dist.all_reduce(self.sum_counts, op=dist.ReduceOp.SUM, group=self.group)
            self.sum_total += self.sum_counts
            fp8.fp8_mu_update(self.mu, self.clean, self.sum_counts, self.n, **self.rule)
        return self.out[:self.hi - self.lo]

    def all_gather(self) -> torch.Tensor:
        """The whole summed gradient (n codes at scale S) on every rank."""
        if not self.collectives:
            return self.out[:self.n]
        full = torch.empty(self.world * self.L, dtype=torch.uint8, device=self.out.device)
        dist.all_gather_into_tensor(full, self.out, group=self.group)
        return full[:self.n]

    def rates(self) -> dict:
        """Underflow and overflow counts of all steps so far, summed over the
        ranks (a host read, for monitoring; every rank must call it, it runs a
        collective).  Under "auto" the sum counts are the running total that
        was already summed over the ranks step by step."""
        auto = self.scaling == "auto"
        c = self.cast_counts.clone() if auto else torch.cat([self.cast_counts, self.sum_counts])
        if self.collectives:
            dist.all_reduce(c, op=dist.ReduceOp.SUM, group=self.group)
        c = (torch.cat([c, self.sum_total]) if auto else c).tolist()
        return dict(cast_underflow=c[0], cast_overflow=c[1], sum_underflow=c[2], sum_overflow=c[3],
                    mu=self.mu.item())
