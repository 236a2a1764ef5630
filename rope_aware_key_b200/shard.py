"""Splitting one cache over several GPUs by whole (layer, KV head) units.

Every unit (layer, KV head, sequence) is scored, selected and compacted on
its own, and the folded weights are per (layer, KV head), so the path
shards with no exchange at all: each rank takes a contiguous range of
layers -- all KV heads and sequences of those layers -- and runs the
ordinary calls on it.  Units are numbered layer-major,
u = (l * H + h) * batch + b, so a layer range is also a contiguous range
of units (its rows of kept indices, counts and compacted K/V) and of weight
rows (l * H + h).

A rank's view of a cache it shares with the others (one process holding the
whole cache, or a cache whose layers each rank has mapped) is the same
descriptor with the K and V bases moved to its first layer and num_layers
cut to its range; nothing else changes, so the library's host checks apply
to each view as they do to the whole.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

from . import Desc, _CacheDesc

_BF16 = 2


def layer_ranges(num_layers: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous layer ranges [l0, l1) for ranks 0..world-1: as even as
    possible, the first num_layers % world ranks one layer longer.  Ranks
    past the layer count get an empty range."""
    if num_layers < 0 or world < 1:
        raise ValueError("num_layers >= 0 and world >= 1")
    base, extra = divmod(num_layers, world)
    out, l0 = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((l0, l0 + n))
        l0 += n
    return out


@dataclasses.dataclass
class Shard:
    """One rank's part of a cache."""
    rank: int
    layers: Tuple[int, int]         # [l0, l1)
    units: Tuple[int, int]          # [u0, u1) in the whole cache's unit order
    weight_rows: Tuple[int, int]    # rows [l0 * H, l1 * H) of the folded weights
    desc: Optional[Desc]            # the rank's view (None for an empty range)


def shard_layers(desc: Desc, rank: int, world: int) -> Shard:
    """Rank `rank`'s layer range of `desc` as its own descriptor."""
    L, H, Bt = desc.num_layers, desc.num_kv_heads, desc.batch
    l0, l1 = layer_ranges(L, world)[rank]
    per_layer = H * Bt
    shard = Shard(rank, (l0, l1), (l0 * per_layer, l1 * per_layer), (l0 * H, l1 * H), None)
    if l1 == l0:
        return shard
    src = desc.raw
    raw = _CacheDesc.from_buffer_copy(src)
    off = l0 * src.stride_layer * _BF16
    raw.k = src.k + off
    raw.v = src.v + off if src.v else None
    raw.num_layers = l1 - l0
    shard.desc = Desc(raw, [desc], (l1 - l0) * per_layer, desc.lens)
    return shard


def addressed_elements(desc: Desc) -> Tuple[int, int]:
    """The bf16 element range [first, last) of K that the descriptor's layers
    span, relative to the K base it was cut from: per layer, stride_layer
    elements starting at layer 0 of the view (the pages of a paged pool, or
    the heads and sequences of a packed one)."""
    raw = desc.raw
    return 0, raw.num_layers * raw.stride_layer


def element_offset(view: Desc, whole: Desc) -> int:
    """Where the view's K base sits in the whole cache, in bf16 elements."""
    d = view.raw.k - whole.raw.k
    if d % _BF16:
        raise ValueError("view not aligned to an element of the whole")
    return d // _BF16


__all__ = ["layer_ranges", "Shard", "shard_layers", "addressed_elements", "element_offset"]
