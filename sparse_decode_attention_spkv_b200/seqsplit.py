"""Decode of sequences whose gated cache is split into slices by position.

When one sequence's cache outgrows a device, it can be spread over several caches --
one per GPU -- each holding the gated rows of a range of positions; the last slice
also holds the window (the ring) and takes the per-token retirements, so the earlier
slices stay fixed while decoding goes on.  Every slice computes the attention over its
own keys alone (``spkv_decode_attn_partial``: fp32 output and log-sum-exp per query
head), the partials are brought together (an all-gather across the ranks that hold
the slices) and combined by their log-sum-exp weights (``spkv_decode_merge``).  The
result is the attention over the whole key set up to rounding: Eq. (3) of
"Self-Pruned Key-Value Attention" (§2.1) factorises over a disjoint union of key sets.

Every step runs in the library's kernels (and, across GPUs, one NCCL all-gather of
B x Hq x (head_dim + 1) floats per rank); this module only allocates buffers and
orders the calls.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import dist as Dist
from . import spkv as S


def split_bounds(ctx: Sequence[int], n_slices: int, window: int) -> List[Tuple[list, list]]:
    """Position ranges of n_slices slices of every batch row: the row's cached prefix
    [0, ctx_b - window) cut into equal parts; the last part is open-ended (it takes the
    rows retired while decoding).  Returns [(lo per row, hi per row or None)] per slice."""
    out = []
    for i in range(n_slices):
        lo, hi = [], []
        for c in ctx:
            n = max(0, int(c) - window)
            lo.append(n * i // n_slices)
            hi.append(None if i == n_slices - 1 else n * (i + 1) // n_slices)
        out.append((lo, hi))
    return out


class SliceDecode:
    """One slice's share of a split decode step: its partial, the exchange of all the
    slices' partials, and the merge.

    ``holds_window``: this slice holds the window (the ring is read; the cache may then
    be None).  On one device, give every slice its own SliceDecode and merge with
    ``merge_local``; across ranks (one slice per rank, rank order = slice order) call
    ``step``, which all-gathers the partials and merges them on every rank."""

    def __init__(self, p, cache: Optional[S.Cache], ring: Optional[S.Ring], holds_window: bool,
                 device, world: int = 1):
        if not S.spkv_decode_attn_partial_supported(p):
            raise S.SpkvError("spkv_decode_attn_partial", S.ERR_UNSUPPORTED)
        self.p, self.cache, self.ring = p, cache, ring
        self.flags = S.SLICE_WINDOW if holds_window else 0
        self.world = world
        self.ws = S.alloc_decode_workspace(p, cache, device)
        self.o_part = torch.empty((p.B, p.Hq, p.head_dim), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((p.B, p.Hq), dtype=torch.float32, device=device)
        if world > 1:
            self.o_all = torch.empty((world, p.B, p.Hq, p.head_dim), dtype=torch.float32,
                                     device=device)
            self.lse_all = torch.empty((world, p.B, p.Hq), dtype=torch.float32, device=device)

    def partial(self, q, t_pos, stream=None):
        """This slice's attention: fills and returns (o_part, lse_part)."""
        S.spkv_decode_attn_partial(self.p, self.cache, self.ring, q, t_pos, self.flags,
                                   self.o_part, self.lse_part, self.ws, stream=stream)
        return self.o_part, self.lse_part

    def step(self, q, t_pos, o, lse=None):
        """Partial, all-gather of every rank's partial, merge into o [B][Hq][d] (and lse)."""
        self.partial(q, t_pos)
        if self.world == 1:
            S.spkv_decode_merge(self.p, 1, self.o_part, self.lse_part, o, lse)
            return o
        Dist.all_gather_partials(self.o_part, self.lse_part, self.o_all, self.lse_all)
        S.spkv_decode_merge(self.p, self.world, self.o_all, self.lse_all, o, lse)
        return o


def merge_local(p, slices: Sequence[SliceDecode], q, t_pos, o, lse=None):
    """All slices on this device: each slice's partial into one stacked buffer, then
    the merge.  Returns o."""
    dev = q.device
    o_parts = torch.empty((len(slices), p.B, p.Hq, p.head_dim), dtype=torch.float32, device=dev)
    lse_parts = torch.empty((len(slices), p.B, p.Hq), dtype=torch.float32, device=dev)
    for i, sl in enumerate(slices):
        S.spkv_decode_attn_partial(p, sl.cache, sl.ring, q, t_pos, sl.flags, o_parts[i],
                                   lse_parts[i], sl.ws)
    S.spkv_decode_merge(p, len(slices), o_parts, lse_parts, o, lse)
    return o
