"""Declarative Attention host logic: a declared mode becomes a keep-page list.

[DA] "[논문리뷰] Language Models Can Control Their Own Attention", section 3, and its abstract
page: generation is split into three declared modes -- global (whole context), focus (one
named region) and local (recent output only) -- and the engine applies the resulting mask at
page granularity by rewriting the block table so that only kept pages reach the attention
kernel. Here the keep list is that rewrite's input: ascending logical page ids, handed to
oda_decode_blockmask, whose address generation performs the logical -> physical rewrite.

Region rules (the pages give no sizes): focus keeps the sink page, the focused region
[offset, offset + focus_len) and the `recent` latest tokens; local keeps the `local_len`
latest tokens; every region keeps each 16-token page it touches.
"""
from __future__ import annotations

import numpy as np

GLOBAL, FOCUS, LOCAL = 0, 1, 2


def _page_ranges(mode: int, t: int, focus_offset: int, focus_len: int, recent: int,
                 local_len: int, block: int):
    last = t // block
    if mode == GLOBAL:
        return [(0, last)]
    if mode == LOCAL:
        return [(max(0, t - local_len + 1) // block, last)]
    if mode == FOCUS:
        lo = min(max(focus_offset, 0), t)
        hi = min(t, focus_offset + focus_len - 1)
        ranges = [(0, 0), (max(0, t - recent + 1) // block, last)]
        if hi >= lo:
            ranges.append((lo // block, hi // block))
        return ranges
    raise ValueError("unknown DA mode %r" % mode)


def keep_pages(mode: int, t: int, focus_offset: int = 0, *, focus_len: int = 32768,
               recent: int = 2048, local_len: int = 4096, block: int = 16) -> np.ndarray:
    """Ascending, de-duplicated logical pages a sequence at position t keeps under `mode`."""
    ranges = sorted(_page_ranges(mode, t, focus_offset, focus_len, recent, local_len, block))
    merged = []
    for a, b in ranges:
        if merged and a <= merged[-1][1] + 1:
            merged[-1][1] = max(merged[-1][1], b)
        else:
            merged.append([a, b])
    if not merged:
        return np.zeros(0, dtype=np.int32)
    return np.concatenate([np.arange(a, b + 1, dtype=np.int32) for a, b in merged])


def keep_lists(draws, positions, max_keep: int, **kw):
    """Keep lists for one step of a batch: int32 [B][max_keep] (unused tail = -1) and int32
    counts [B]. draws[b] has .mode and .focus_offset; positions[b] is the current t."""
    B = len(positions)
    out = np.full((B, max_keep), -1, dtype=np.int32)
    counts = np.zeros(B, dtype=np.int32)
    for b, (d, t) in enumerate(zip(draws, positions)):
        k = keep_pages(d.mode, t, d.focus_offset, **kw)
        if k.size > max_keep:
            raise ValueError("keep list of %d pages exceeds max_keep=%d" % (k.size, max_keep))
        out[b, :k.size] = k
        counts[b] = k.size
    return out, counts
