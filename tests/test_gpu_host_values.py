"""V in pinned host memory (mapped into the device), for out-of-place
compaction: the gather reads only the kept V rows over the bus.  Results must
equal, bit for bit, those with V in device memory, on the three-kernel path
and on the single-kernel step; in-place compaction and unpinned host memory
are refused before anything is launched."""
import numpy as np
import pytest
import torch

import gen
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def tri():
    import rope_aware_key_b200 as t
    return t


def run(t, d, w, B, mode, fused, units):
    kept = torch.full((units, B), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((units,), -1, dtype=torch.int32, device=DEV)
    ko = torch.zeros((units, B, 128), dtype=torch.bfloat16, device=DEV)
    vo = torch.zeros_like(ko)
    if fused:
        ws = torch.empty(t.workspace_size(d, B), dtype=torch.uint8, device=DEV)
        t.compress(d, w, B, mode, kept, cnt, ko, vo, ws)
    else:
        sc = torch.empty((units, t.score_row_stride(d)), dtype=torch.float32, device=DEV)
        t.score_keys(d, w, sc)
        t.select_topk(d, sc, B, kept, cnt)
        t.compact_kv(d, kept, cnt, B, mode, ko, vo)
    assert t.read_device_status(clear=True) == 0
    torch.cuda.synchronize()
    return kept, cnt, ko, vo


@pytest.mark.parametrize("layout,fused", [("contig", False), ("contig", True), ("ragged", False)])
def test_values_in_host_memory_give_the_same_compaction(layout, fused):
    t = tri()
    if layout == "contig":
        wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=4, seq_len=4096, budget=700)
        cache = gen.make_cache(wl, seed=61, device=DEV)
    else:
        wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=3, budget=300)
        cache = gen.make_cache(wl, seed=62, device=DEV, lens=[900, 5000, 77])
    d = parity.make_desc(cache)
    hv = cache.v.cpu().pin_memory()
    if layout == "contig":
        dh = t.desc_contig(cache.k, hv)
    else:
        dh = t.desc_ragged(cache.k, hv, cache.cu_seqlens.cpu().tolist())
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = t.fold_weights(qc, wl.theta, wl.offsets)
    B = wl.budget
    ref = run(t, d, w, B, t.COMPACT_OUT_OF_PLACE, fused, d.units)
    got = run(t, dh, w, B, t.COMPACT_OUT_OF_PLACE, fused, d.units)
    assert torch.equal(got[1], ref[1])
    valid = torch.arange(B, device=DEV)[None, :] < ref[1][:, None]
    assert torch.equal(torch.where(valid, got[0], 0), torch.where(valid, ref[0], 0))
    v3 = valid[:, :, None]
    for a, b in ((got[2], ref[2]), (got[3], ref[3])):
        assert torch.equal(torch.where(v3, a.view(torch.int16), 0), torch.where(v3, b.view(torch.int16), 0))
    # and against the cache itself: V rows of the kept keys of one unit
    u = d.units - 1
    n = int(ref[1][u])
    b, lh = u % wl.batch, u // wl.batch
    rows = gen.unit_rows(cache, cache.v, lh // wl.num_kv_heads, lh % wl.num_kv_heads, b)
    np.testing.assert_array_equal(parity.bits16(got[3][u, :n]), parity.bits16(rows)[got[0][u, :n].cpu().numpy()])


def test_values_in_host_memory_refused_where_they_would_be_written_or_are_not_mapped():
    t = tri()
    wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=2, seq_len=3000, budget=500)
    cache = gen.make_cache(wl, seed=63, device=DEV)
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = t.fold_weights(qc, wl.theta, wl.offsets)
    B = wl.budget
    kept = torch.empty((2, B), dtype=torch.int32, device=DEV)
    cnt = torch.empty((2,), dtype=torch.int32, device=DEV)
    pinned = t.desc_contig(cache.k, cache.v.cpu().pin_memory())
    plain = t.desc_contig(cache.k, cache.v.cpu())
    ws = torch.empty(t.workspace_size(pinned, B), dtype=torch.uint8, device=DEV)
    n0 = t.kernel_launches()
    with pytest.raises(t.TriError) as e:                # in place would write the host copy
        t.compress(pinned, w, B, t.COMPACT_IN_PLACE_HOLEFILL, kept, cnt, None, None, ws)
    assert e.value.status == 1
    ko = torch.empty((2, B, 128), dtype=torch.bfloat16, device=DEV)
    vo = torch.empty_like(ko)
    with pytest.raises(t.TriError) as e:                # pageable host memory: not mapped
        t.compress(plain, w, B, t.COMPACT_OUT_OF_PLACE, kept, cnt, ko, vo, ws)
    assert e.value.status == 1
    assert t.kernel_launches() == n0
