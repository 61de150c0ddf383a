"""Context-parallel Full decode: the history of every sequence is cut into page-aligned
position ranges, one per rank (one GPU each); a rank keeps the KV pages of its range only and
attends them with oda_decode under the SHARD rule, producing a normalised partial (O, LSE)
per (sequence, query head). The partials of all ranks are exchanged with one all-gather over
the process group (NCCL over NVLink on GPUs; 8.3 KB per sequence for 16 query heads) and
combined on every rank by oda_merge_partials, so every rank ends with the Full result.

The gate is computed on every rank from replicated inputs, so all ranks take the same branch
and issue the same collectives in the same order. The commit of slot t happens on the one
rank whose range holds t."""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import oda

OPEN_END = 1 << 30   # the last range runs to the end of every sequence


def shard_bounds(capacity_tokens: int, world: int) -> List[Tuple[int, int]]:
    """Page-aligned [lo, hi) position ranges, one per rank, splitting 0..capacity_tokens-1 as
    evenly as whole 16-token pages allow; the last range is open-ended (hi = OPEN_END) so
    that tokens appended during decoding land on the last rank."""
    if world < 1 or capacity_tokens < 0:
        raise ValueError("world >= 1 and capacity_tokens >= 0 required")
    pages = (capacity_tokens + 15) // 16
    cuts = [16 * (pages * r // world) for r in range(world)] + [OPEN_END]
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def gather_partials(o_part: torch.Tensor, lse_part: torch.Tensor, group=None):
    """All-gather every rank's (O, LSE) partial: returns ([R][B][Hq][128], [R][B][Hq]) in rank
    order. One collective per tensor, contiguous outputs."""
    world = dist.get_world_size(group)
    # outputs are the rank blocks concatenated along dim 0, the layout every backend takes
    o_all = torch.empty((world * o_part.shape[0],) + tuple(o_part.shape[1:]), dtype=o_part.dtype,
                        device=o_part.device)
    l_all = torch.empty((world * lse_part.shape[0],) + tuple(lse_part.shape[1:]),
                        dtype=lse_part.dtype, device=lse_part.device)
    dist.all_gather_into_tensor(o_all, o_part.contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse_part.contiguous(), group=group)
    return (o_all.view((world,) + tuple(o_part.shape)),
            l_all.view((world,) + tuple(lse_part.shape)))


class ContextParallelFull:
    """Full decode of one layer over a history sharded across the ranks of `group`.

    kv: this rank's oda_kv (its own pages; block-table entries outside the rank's range are
    never read); bounds: this rank's (lo, hi) from shard_bounds."""

    def __init__(self, batch: int, num_q_heads: int, bounds: Tuple[int, int], ws: torch.Tensor,
                 group=None):
        self.lo, self.hi = bounds
        self.group = group
        dev = ws.device
        self.ws = ws
        self.o_part = torch.empty((batch, num_q_heads, 128), dtype=torch.float32, device=dev)
        self.l_part = torch.empty((batch, num_q_heads), dtype=torch.float32, device=dev)

    def __call__(self, kv, q, scale: float, out, gate: Optional[torch.Tensor] = None,
                 k_new=None, v_new=None, lse=None, stream=None):
        vis = oda.shard_visibility(self.lo, self.hi, gate=gate)
        oda.oda_decode(kv, vis, q, scale, self.o_part, self.ws, k_new=k_new, v_new=v_new,
                       lse=self.l_part, stream=stream)
        o_all, l_all = gather_partials(self.o_part, self.l_part, self.group)
        oda.oda_merge_partials(o_all, l_all, out, gate=gate, lse=lse, stream=stream)
        return out
