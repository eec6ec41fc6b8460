"""Token-sharded decode over several ranks, one process per GPU.

The pages' capacity claim -- LLaMA-7B with up to 10 million tokens of context across 8 GPUs
(study.space summary; phantomic12 research note, consequence claim) -- needs each sequence's
cache split across devices.  Every rank keeps one contiguous range of each sequence's tokens in
a cache of its own (quantized and key-calibrated on that range), and per decode step and layer:

  1. ``kvq_decode_partial`` over its range, at the range's absolute positions -> (M, L, o);
  2. one all-gather of every rank's (M, L, o) through ``torch.distributed`` (NCCL on GPUs);
  3. ``kvq_merge_partials`` over the gathered partials -> the attention output, on every rank.

The exchange is (8 + 4*D) bytes per (sequence, query head) per rank; nothing else crosses ranks.
New tokens are appended by the rank holding the end of the sequences (the last rank).  This
module only plans ranges and moves tensors; the arithmetic is the library's.
"""
from __future__ import annotations

from . import kvq as K

CHUNK = K.CHUNK


def token_ranges(T: int, world: int):
    """Contiguous [lo, hi) ranges of T tokens over `world` ranks, 64-token aligned (the last
    may be short; trailing ranks may be empty when T is small)."""
    per = (-(-T // world) + CHUNK - 1) // CHUNK * CHUNK
    return [(min(T, r * per), min(T, (r + 1) * per)) for r in range(world)]


def append_rank(world: int) -> int:
    """The rank that appends new tokens: the one holding the end of the sequences."""
    return world - 1


class PartialExchange:
    """The all-gather of step 2: every rank's (M, L) [B, Hq, 2] and o [B, Hq, D] into
    [world, ...] buffers, views of which are handed to the collective in rank order."""

    def __init__(self, B: int, Hq: int, D: int, world: int, device, dtype=None, group=None):
        import torch
        dtype = dtype or torch.float32
        self.world = world
        self.group = group
        self.ml = torch.empty((world, B, Hq, 2), dtype=dtype, device=device)
        self.o = torch.empty((world, B, Hq, D), dtype=dtype, device=device)

    def __call__(self, ml, o):
        import torch.distributed as dist
        if self.world == 1:
            self.ml[0].copy_(ml)
            self.o[0].copy_(o)
        else:
            dist.all_gather(list(self.ml.unbind(0)), ml.contiguous(), group=self.group)
            dist.all_gather(list(self.o.unbind(0)), o.contiguous(), group=self.group)
        return self.ml, self.o


class ShardedDecode:
    """Steps 1-3 for one rank: local partial, exchange, merge."""

    def __init__(self, cfg, world: int, rank: int, device, group=None):
        import torch
        self.cfg, self.world, self.rank = cfg, world, rank
        self.ml = torch.empty((cfg.B, cfg.Hq, 2), dtype=torch.float32, device=device)
        self.o = torch.empty((cfg.B, cfg.Hq, cfg.D), dtype=torch.float32, device=device)
        self.exchange = PartialExchange(cfg.B, cfg.Hq, cfg.D, world, device, group=group)

    def __call__(self, cache, cbK, cbV, q, qpos, max_len: int, pos_offset: int, out, workspace,
                 splits: int = 0):
        K.kvq_decode_partial(cache, cbK, cbV, q, qpos, max_len, pos_offset, self.ml, self.o,
                             workspace, splits)
        ml_all, o_all = self.exchange(self.ml, self.o)
        K.kvq_merge_partials(self.cfg, self.world, ml_all, o_all, out)
        return out
