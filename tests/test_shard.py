"""Splitting one cache over ranks by whole layers (rope_aware_key_b200.shard),
on CPU: two gloo ranks each cut their view of the same cache, and the views
together must cover every unit exactly once, address disjoint parts of K
whose union is the whole cache, and give the sizes the library's host checks
compute for the whole.  No GPU and no kernel: the library calls used here
(row stride, workspace size) are host-only."""
import ctypes
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_layer_ranges_partition():
    from rope_aware_key_b200.shard import layer_ranges
    for L in (1, 2, 5, 36, 80):
        for world in (1, 2, 3, 4, 8):
            r = layer_ranges(L, world)
            assert len(r) == world and r[0][0] == 0 and r[-1][1] == L
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [b - a for a, b in r]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    assert layer_ranges(2, 3) == [(0, 1), (1, 2), (2, 2)]
    with pytest.raises(ValueError):
        layer_ranges(4, 0)


def _caches():
    """Host descriptors of one cache in each layout (CPU tensors or fake
    aligned addresses: nothing is dereferenced)."""
    import rope_aware_key_b200 as tri
    out = {}
    k = torch.zeros((5, 3, 2, 40, 128), dtype=torch.bfloat16)
    out["contig"] = tri.desc_contig(k, k.clone())
    kr = torch.zeros((5, 2, 90, 128), dtype=torch.bfloat16)
    out["ragged"] = tri.desc_ragged(kr, kr.clone(), [0, 30, 30, 90])
    lens = (tri._i32_host([40, 17, 64]))
    raw = tri._CacheDesc(layout=tri.LAYOUT_PAGED, num_layers=5, num_kv_heads=4, head_dim=128, batch=3,
                         k=0x100000, v=0x900000, stride_layer=20 * 16 * 4 * 128, stride_block=16 * 4 * 128,
                         seq_lens=ctypes.cast(lens, ctypes.POINTER(ctypes.c_int32)), block_table=0x10000,
                         max_blocks_per_seq=4, block_size=16, num_blocks=20)
    out["paged"] = tri.Desc(raw, [lens], 5 * 4 * 3, [40, 17, 64])
    return out


def _summaries(rank, world):
    import rope_aware_key_b200 as tri
    from rope_aware_key_b200.shard import addressed_elements, element_offset, shard_layers
    L = tri.lib()
    res = {}
    for name, whole in _caches().items():
        sh = shard_layers(whole, rank, world)
        d = sh.desc
        off = element_offset(d, whole)
        first, last = addressed_elements(d)
        n = ctypes.c_size_t(0)
        assert L.tri_workspace_size(d.ref, 8, ctypes.byref(n)) == 0
        res[name] = dict(layers=sh.layers, units=sh.units, weight_rows=sh.weight_rows, unit_count=d.units,
                         elems=(off + first, off + last), v_off=(d.raw.v - whole.raw.v) // 2,
                         workspace=n.value, stride=L.tri_score_row_stride(d.ref))
    return res


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world)
    try:
        mine = _summaries(rank, world)
        every = [None] * world
        torch.distributed.all_gather_object(every, mine)
        out[rank] = every
    finally:
        torch.distributed.destroy_process_group()


def test_gloo_two_ranks_cover_the_cache_once():
    import rope_aware_key_b200 as tri
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == out[1]                       # both ranks agree on the plan
    per_rank = out[0]
    L = tri.lib()
    for name, whole in _caches().items():
        H, Bt, nl = whole.num_kv_heads, whole.batch, whole.num_layers
        parts = [p[name] for p in per_rank]
        # layers 0..2 and 3..4 of 5
        assert [p["layers"] for p in parts] == [(0, 3), (3, 5)]
        # every unit exactly once, in the whole cache's order
        units = sorted(u for p in parts for u in range(*p["units"]))
        assert units == list(range(nl * H * Bt))
        assert sum(p["unit_count"] for p in parts) == whole.units
        assert sorted(r for p in parts for r in range(*p["weight_rows"])) == list(range(nl * H))
        # disjoint element ranges of K whose union is the whole cache's; V moves with K
        spans = sorted(p["elems"] for p in parts)
        assert spans[0][0] == 0 and spans[-1][1] == nl * whole.raw.stride_layer
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        assert all(p["v_off"] == p["elems"][0] for p in parts)
        # the sizes the host checks compute: same score rows, workspaces adding up
        n = ctypes.c_size_t(0)
        assert L.tri_workspace_size(whole.ref, 8, ctypes.byref(n)) == 0
        assert sum(p["workspace"] - 256 for p in parts) == n.value - 256
        assert all(p["stride"] == L.tri_score_row_stride(whole.ref) for p in parts)


def test_view_rows_are_the_whole_caches_rows():
    """Row (l', h, b, i) of rank 1's view is row (l0 + l', h, b, i) of the whole."""
    import rope_aware_key_b200 as tri
    from rope_aware_key_b200.shard import element_offset, shard_layers
    k = torch.randn((5, 3, 2, 40, 128), generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    whole = tri.desc_contig(k, k)
    sh = shard_layers(whole, 1, 2)
    off = element_offset(sh.desc, whole)
    raw = sh.desc.raw
    flat = k.view(-1)
    for (lp, h, b, i) in [(0, 0, 0, 0), (1, 2, 1, 39), (0, 1, 1, 7)]:
        e_view = off + lp * raw.stride_layer + h * raw.stride_head + b * raw.stride_seq + i * 128
        assert torch.equal(flat[e_view:e_view + 128], k[sh.layers[0] + lp, h, b, i])
        u_view = (lp * raw.num_kv_heads + h) * raw.batch + b
        assert sh.units[0] + u_view == ((sh.layers[0] + lp) * 3 + h) * 2 + b


def test_empty_range_when_ranks_outnumber_layers():
    import rope_aware_key_b200 as tri
    from rope_aware_key_b200.shard import shard_layers
    k = torch.zeros((2, 1, 1, 8, 128), dtype=torch.bfloat16)
    whole = tri.desc_contig(k, k)
    sh = shard_layers(whole, 2, 3)
    assert sh.desc is None and sh.units[0] == sh.units[1] == 2
