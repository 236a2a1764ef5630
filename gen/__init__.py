"""Seeded synthetic inputs for the score -> select -> compact path.

This module only draws random numbers and lays them out in the cache layouts
the library accepts.  It holds none of the method's arithmetic (no band
frequencies, no folding, no scoring, no selection, no compaction), so both
the CUDA path (tests, bench) and the CPU oracle can take their inputs from it
without sharing any of the computation.

Recipe (one cache per workload and seed):

* key center  c[l][h]  ~ N(0, 1)^d            fp32, drawn on the CPU
* query center q[l][h] ~ N(0, 1)^d            fp32, drawn on the CPU
* key i of unit (l, h, b): k = c[l][h] + sigma * N(0, 1)^d; with probability
  ``outlier_p`` (a Bernoulli draw per key) the whole vector is scaled by
  ``outlier_scale`` before the bf16 round-to-nearest-even
* value rows  v ~ N(0, 1)^d                     bf16
* ragged / paged sequence lengths ~ U{len_lo .. len_hi} (integers, inclusive)
* paged caches: physical block ids are a seeded random permutation, so a
  sequence's pages are scattered over the pool

Keys and values are drawn per (layer, sequence) with a torch generator seeded
from ``sub_seed(seed, tag, layer, seq)``, so one layer can be regenerated on
its own.  The stream depends on the device type of the generator (torch's CPU
and CUDA generators differ); every consumer hands the very same tensors to
both sides, so that never matters for parity.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import torch

_MASK64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    """One SplitMix64 output step (Steele, Lea and Flood, OOPSLA 2014)."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


_TAGS = {"key_center": 1, "query_center": 2, "K": 3, "V": 4, "lens": 5,
         "blocks": 6, "append_K": 7, "append_V": 8, "positions": 9}


def sub_seed(seed: int, tag: str, *idx: int) -> int:
    """Derive an independent 63-bit generator seed for (seed, tag, idx...)."""
    h = _splitmix64(seed & _MASK64)
    h = _splitmix64(h ^ _TAGS[tag])
    for i in idx:
        h = _splitmix64(h ^ (i & _MASK64))
    return h & ((1 << 63) - 1)


def _gen(device, s: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def geometric_offsets(lo_exp: int = 0, hi_exp: int = 16) -> List[float]:
    """The offset schedule {2^lo .. 2^hi} as floats."""
    return [float(2 ** e) for e in range(lo_exp, hi_exp + 1)]


def uniform_offsets(m: int) -> List[float]:
    """The offset schedule {1, 2, ..., m} as floats."""
    return [float(i) for i in range(1, m + 1)]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_layers: int
    num_kv_heads: int
    head_dim: int
    theta: float
    offsets: tuple
    budget: int
    layout: str                 # "contig" | "ragged" | "paged"
    batch: int = 1
    seq_len: int = 0            # contig: keys per unit
    len_lo: int = 0             # ragged / paged: length range (inclusive)
    len_hi: int = 0
    block_size: int = 16
    sigma: float = 0.3
    outlier_p: float = 0.01
    outlier_scale: float = 5.0
    delta0: float = 0.0
    spare_blocks_per_seq: int = 0   # paged: free pages for appended tokens

    @property
    def units(self) -> int:
        return self.num_layers * self.num_kv_heads * self.batch


_GEO17 = tuple(geometric_offsets(0, 16))

WORKLOADS: Dict[str, Workload] = {
    # single head, 4096 keys, theta 1e4, B = 512
    "tiny": Workload("tiny", 1, 1, 128, 1e4, _GEO17, 512, "contig",
                     batch=1, seq_len=4096),
    # one Qwen3-8B-shaped layer: 8 KV heads x 32768 keys, B = 2048
    "qwen3_layer": Workload("qwen3_layer", 1, 8, 128, 1e6, _GEO17, 2048,
                            "contig", batch=1, seq_len=32768),
    # full Qwen3-8B-shaped cache, 36 layers x 8 heads x 32768 keys, batch 1
    "qwen3_full": Workload("qwen3_full", 36, 8, 128, 1e6, _GEO17, 2048,
                           "contig", batch=1, seq_len=32768),
    # 8 of those 36 layers: a smaller case of the same shape (profiling)
    "qwen3_8layers": Workload("qwen3_8layers", 8, 8, 128, 1e6, _GEO17, 2048, "contig",
                              batch=1, seq_len=32768),
    # 36 x 8, batch 8 ragged sequences of U{8192..32768} tokens
    "qwen3_ragged": Workload("qwen3_ragged", 36, 8, 128, 1e6, _GEO17, 2048,
                             "ragged", batch=8, len_lo=8192, len_hi=32768),
    # Llama3-70B-shaped long cache, uniform schedule {1..1024}, B = 12000
    "llama3_long": Workload("llama3_long", 80, 8, 128, 5e5,
                            tuple(uniform_offsets(1024)), 12000, "contig",
                            batch=1, seq_len=131072, sigma=0.5),
    # Qwen2.5-7B-shaped paged cache, 64 sequences, 16-token pages
    "qwen25_paged": Workload("qwen25_paged", 28, 4, 128, 1e6, _GEO17, 2048,
                             "paged", batch=64, len_lo=8192, len_hi=32768,
                             block_size=16, spare_blocks_per_seq=8),
    # 1 of those 28 layers: a smaller case of the same shape (profiling)
    "qwen25_paged_1layer": Workload("qwen25_paged_1layer", 1, 4, 128, 1e6, _GEO17, 2048,
                                    "paged", batch=64, len_lo=8192, len_hi=32768,
                                    block_size=16, spare_blocks_per_seq=8),
}


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of ``wl`` with some fields replaced (used for small test cases)."""
    return dataclasses.replace(wl, **changes)


# ---------------------------------------------------------------- draws

def seq_lengths(wl: Workload, seed: int) -> List[int]:
    """Per-sequence key counts."""
    if wl.layout == "contig":
        return [wl.seq_len] * wl.batch
    g = _gen("cpu", sub_seed(seed, "lens"))
    n = torch.randint(wl.len_lo, wl.len_hi + 1, (wl.batch,), generator=g)
    return [int(x) for x in n]


def centers(wl: Workload, seed: int):
    """(key_center, query_center), each fp32 [L][H][d] on the CPU."""
    shape = (wl.num_layers, wl.num_kv_heads, wl.head_dim)
    kc = torch.randn(shape, generator=_gen("cpu", sub_seed(seed, "key_center")))
    qc = torch.randn(shape, generator=_gen("cpu", sub_seed(seed, "query_center")))
    return kc, qc


def draw_keys(wl: Workload, seed: int, layer: int, seq: int, n: int,
              key_center_l: torch.Tensor, device, tag: str = "K") -> torch.Tensor:
    """bf16 keys [H][n][d] of layer ``layer``, sequence ``seq``."""
    H, d = wl.num_kv_heads, wl.head_dim
    g = _gen(device, sub_seed(seed, tag, layer, seq))
    x = torch.randn((H, n, d), generator=g, device=device)
    x.mul_(wl.sigma).add_(key_center_l.to(device).view(H, 1, d))
    u = torch.rand((H, n, 1), generator=g, device=device)
    scale = torch.where(u < wl.outlier_p, wl.outlier_scale, 1.0)
    x.mul_(scale)
    return x.to(torch.bfloat16)


def draw_values(wl: Workload, seed: int, layer: int, seq: int, n: int,
                device, tag: str = "V") -> torch.Tensor:
    """bf16 values [H][n][d] of layer ``layer``, sequence ``seq``."""
    H, d = wl.num_kv_heads, wl.head_dim
    g = _gen(device, sub_seed(seed, tag, layer, seq))
    return torch.randn((H, n, d), generator=g, device=device).to(torch.bfloat16)


# ---------------------------------------------------------------- caches

@dataclasses.dataclass
class Cache:
    """A synthetic cache and its metadata (all tensors on ``device``)."""
    wl: Workload
    seed: int
    lens: List[int]
    key_center: torch.Tensor          # fp32 [L][H][d] (CPU)
    query_center: torch.Tensor        # fp32 [L][H][d] (CPU)
    k: torch.Tensor
    v: torch.Tensor
    cu_seqlens: Optional[torch.Tensor] = None    # ragged, int32 [batch+1]
    block_table: Optional[torch.Tensor] = None   # paged, int32 [batch][max_blocks]
    seq_lens: Optional[torch.Tensor] = None      # paged, int32 [batch]
    free_blocks: Optional[List[int]] = None      # paged, unused physical pages
    layer0: int = 0                              # first layer of the full cache that this one holds

    @property
    def max_len(self) -> int:
        return max(self.lens) if self.lens else 0


def make_cache(wl: Workload, seed: int, device="cpu", with_values: bool = True,
               lens: Optional[Sequence[int]] = None, layer_range: Optional[Sequence[int]] = None) -> Cache:
    """Draw a full cache for ``wl`` in its layout.

    contig: K, V bf16 [L][H][batch][N][d]
    ragged: K, V bf16 [L][H][T][d] with cu_seqlens (int32, prefix sums of lens)
    paged:  K, V bf16 [L][num_blocks][block_size][H][d] with an int32 block table

    ``layer_range`` = (l0, l1) draws only layers l0 .. l1-1 of that cache --
    the very same numbers, since every layer has its own generator seeds --
    as a cache of l1 - l0 layers (its workload's num_layers cut to match).
    """
    l0, l1 = (0, wl.num_layers) if layer_range is None else (int(layer_range[0]), int(layer_range[1]))
    assert 0 <= l0 <= l1 <= wl.num_layers
    H, d = wl.num_kv_heads, wl.head_dim
    lens = list(lens) if lens is not None else seq_lengths(wl, seed)
    kc, qc = centers(wl, seed)
    kc, qc = kc[l0:l1].contiguous(), qc[l0:l1].contiguous()
    if layer_range is not None:
        wl = scaled(wl, num_layers=l1 - l0)
    L = wl.num_layers
    c = Cache(wl, seed, lens, kc, qc, None, None, layer0=l0)

    if wl.layout == "contig":
        N = wl.seq_len if lens is None else max(lens)
        assert all(n == N for n in lens)
        c.k = torch.empty((L, H, wl.batch, N, d), dtype=torch.bfloat16, device=device)
        c.v = torch.empty_like(c.k) if with_values else None
        for l in range(L):
            for b in range(wl.batch):
                c.k[l, :, b] = draw_keys(wl, seed, l0 + l, b, N, kc[l], device)
                if with_values:
                    c.v[l, :, b] = draw_values(wl, seed, l0 + l, b, N, device)
    elif wl.layout == "ragged":
        cu = [0]
        for n in lens:
            cu.append(cu[-1] + n)
        T = cu[-1]
        c.k = torch.empty((L, H, T, d), dtype=torch.bfloat16, device=device)
        c.v = torch.empty_like(c.k) if with_values else None
        for l in range(L):
            for b, n in enumerate(lens):
                c.k[l, :, cu[b]:cu[b + 1]] = draw_keys(wl, seed, l0 + l, b, n, kc[l], device)
                if with_values:
                    c.v[l, :, cu[b]:cu[b + 1]] = draw_values(wl, seed, l0 + l, b, n, device)
        c.cu_seqlens = torch.tensor(cu, dtype=torch.int32, device=device)
    elif wl.layout == "paged":
        bs = wl.block_size
        need = [(n + bs - 1) // bs for n in lens]
        max_blocks = max(need) + wl.spare_blocks_per_seq if need else 1
        num_blocks = sum(need) + wl.spare_blocks_per_seq * wl.batch
        perm = torch.randperm(num_blocks, generator=_gen("cpu", sub_seed(seed, "blocks")))
        perm = [int(x) for x in perm]
        table = torch.zeros((wl.batch, max_blocks), dtype=torch.int32)
        pos = 0
        for b, nb in enumerate(need):
            table[b, :nb] = torch.tensor(perm[pos:pos + nb], dtype=torch.int32)
            pos += nb
        c.free_blocks = perm[pos:]
        c.block_table = table.to(device)
        c.seq_lens = torch.tensor(lens, dtype=torch.int32, device=device)
        c.k = torch.zeros((L, num_blocks, bs, H, d), dtype=torch.bfloat16, device=device)
        c.v = torch.zeros_like(c.k) if with_values else None
        for l in range(L):
            for b, n in enumerate(lens):
                slots = paged_slots(table[b], n, bs).to(device)
                kf = c.k[l].view(num_blocks * bs, H, d)
                kf[slots] = draw_keys(wl, seed, l0 + l, b, n, kc[l], device).permute(1, 0, 2)
                if with_values:
                    vf = c.v[l].view(num_blocks * bs, H, d)
                    vf[slots] = draw_values(wl, seed, l0 + l, b, n, device).permute(1, 0, 2)
    else:
        raise ValueError(f"unknown layout {wl.layout!r}")
    return c


def key_positions(c: Cache, seed: int, stride: int, spread: int = 4, device=None):
    """Positions of a pre-RoPE cache that was compacted before: for every unit
    (order layer, head, sequence) its lens[b] keys keep a sorted random
    sample of distinct original positions in [0, spread * lens[b]).  Returns
    (int32 [units][stride], padding -1; the query position of each
    sequence, spread * lens[b])."""
    wl = c.wl
    device = device or c.k.device
    units = wl.num_layers * wl.num_kv_heads * wl.batch
    pos = torch.full((units, stride), -1, dtype=torch.int32, device=device)
    for l in range(wl.num_layers):
        for h in range(wl.num_kv_heads):
            for b, n in enumerate(c.lens):
                if n == 0:
                    continue
                g = _gen(device, sub_seed(seed, "positions", c.layer0 + l, h, b))
                pick = torch.randperm(spread * n, generator=g, device=device)[:n]
                u = (l * wl.num_kv_heads + h) * wl.batch + b
                pos[u, :n] = torch.sort(pick).values.to(torch.int32)
    return pos, [spread * n for n in c.lens]


def paged_slots(table_row: torch.Tensor, n: int, bs: int) -> torch.Tensor:
    """Flat page-pool slot (block * bs + offset) of tokens 0..n-1 of one sequence."""
    i = torch.arange(n, dtype=torch.int64)
    return table_row.to(torch.int64).cpu()[i // bs] * bs + i % bs


def unit_rows(c: Cache, tensor: torch.Tensor, layer: int, head: int, seq: int) -> torch.Tensor:
    """The rows [n][d] of one unit, in key order, as a view or a gathered copy."""
    wl = c.wl
    n = c.lens[seq]
    if wl.layout == "contig":
        return tensor[layer, head, seq, :n]
    if wl.layout == "ragged":
        cu = c.cu_seqlens.cpu()
        return tensor[layer, head, int(cu[seq]):int(cu[seq + 1])]
    bs = wl.block_size
    slots = paged_slots(c.block_table[seq].cpu(), n, bs).to(tensor.device)
    flat = tensor[layer].reshape(-1, wl.num_kv_heads, wl.head_dim)
    return flat[slots, head]


def append_tokens(c: Cache, n_new: int, step: int) -> None:
    """Paged: append ``n_new`` freshly drawn tokens to every sequence.

    Pages come from ``c.free_blocks``; sequence lengths and the block table are
    updated in place.  Used to drive repeated compression events.
    """
    wl = c.wl
    assert wl.layout == "paged"
    bs, H, d = wl.block_size, wl.num_kv_heads, wl.head_dim
    dev = c.k.device
    table = c.block_table.cpu()
    for b in range(wl.batch):
        n0 = c.lens[b]
        n1 = n0 + n_new
        nb0, nb1 = (n0 + bs - 1) // bs, (n1 + bs - 1) // bs
        for j in range(nb0, nb1):
            if j >= table.shape[1]:
                raise RuntimeError("block table too narrow for the append")
            table[b, j] = c.free_blocks.pop()
        row = table[b]
        slots_all = paged_slots(row, n1, bs)
        slots = slots_all[n0:n1].to(dev)
        for l in range(wl.num_layers):
            kf = c.k[l].view(-1, H, d)
            kf[slots] = draw_keys(wl, c.seed, c.layer0 + l, (step << 16) | b, n_new,
                                  c.key_center[l], dev, tag="append_K").permute(1, 0, 2)
            if c.v is not None:
                vf = c.v[l].view(-1, H, d)
                vf[slots] = draw_values(wl, c.seed, c.layer0 + l, (step << 16) | b, n_new, dev,
                                        tag="append_V").permute(1, 0, 2)
        c.lens[b] = n1
    c.block_table = table.to(dev)
    c.seq_lens = torch.tensor(c.lens, dtype=torch.int32, device=dev)


def release_tail_blocks(c: Cache, new_lens: Sequence[int]) -> None:
    """Paged: shrink sequences to ``new_lens`` and return whole tail pages."""
    bs = c.wl.block_size
    table = c.block_table.cpu()
    for b, n in enumerate(new_lens):
        keep = (n + bs - 1) // bs
        had = (c.lens[b] + bs - 1) // bs
        for j in range(keep, had):
            c.free_blocks.append(int(table[b, j]))
            table[b, j] = 0
        c.lens[b] = n
    c.block_table = table.to(c.k.device)
    c.seq_lens = torch.tensor(c.lens, dtype=torch.int32, device=c.k.device)
