"""tri_compress_noalloc, the entry point for callers that cannot allocate
device memory (for instance an engine whose KV-cache pool already holds
nearly all free HBM): its score scratch is an array compiled into the
library instead of a caller-provided workspace.  It must give exactly what
tri_compress gives -- the kept indices, their counts and the compacted K/V
are integer and bit-copy results, so the bar is equality -- and it must keep
doing so on a second call that reuses the scratch left by the first.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import pytest
import torch

import gen
from tests import parity

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    import rope_aware_key_b200 as tri
    fn = lib.tri_compress_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(tri._CacheDesc), P, ctypes.c_int, ctypes.c_int, P, P, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _call_noalloc(fn, tri, d, w, B, mode, kept, cnt, ko, vo):
    P = ctypes.c_void_p
    st = fn(d.ref, P(w.data_ptr()), B, mode, P(kept.data_ptr()), P(cnt.data_ptr()),
            P(ko.data_ptr() if ko is not None else 0), P(vo.data_ptr() if vo is not None else 0),
            P(torch.cuda.current_stream().cuda_stream))
    assert st == 0, tri.TriError(st, "tri_compress_noalloc")


def test_noalloc_matches_compress_on_two_calls():
    import rope_aware_key_b200 as tri
    lib = tri.lib()
    fn = _noalloc(lib)
    dev = torch.device("cuda:0")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    # in a row: a full 8-head layer (three kernels); a smaller ragged cache,
    # which must not be affected by the scores the first call left behind; a
    # cache of 4 units x 4096 keys, which takes the single-kernel step (one
    # cluster per unit, scores in the shared array); a paged cache compacted
    # in place (three kernels, hole fill); and a paged cache whose rows move
    # few keys (two kernels: the score, then the selection with the fill)
    cases = [
        (gen.WORKLOADS["qwen3_layer"], None, 1, tri.COMPACT_OUT_OF_PLACE, 3),
        (gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=4, batch=3, budget=300),
         [900, 4000, 77], 2, tri.COMPACT_OUT_OF_PLACE, 3),
        (gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=4, seq_len=4096, budget=512), None, 3,
         tri.COMPACT_OUT_OF_PLACE, 1 if 4 * 16 <= sms else 3),
        (gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=4, batch=3, budget=2048,
                    spare_blocks_per_seq=1), [2176, 5000, 300], 4, tri.COMPACT_IN_PLACE_HOLEFILL, 3),
        (gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=4, batch=3, budget=2048,
                    spare_blocks_per_seq=1), [2176, 2100, 300], 5, tri.COMPACT_IN_PLACE_HOLEFILL, 2),
    ]
    for wl, lens, seed, mode, launches in cases:
        in_place = mode == tri.COMPACT_IN_PLACE_HOLEFILL
        cache = gen.make_cache(wl, seed=seed, device=dev, lens=lens)
        twin = gen.make_cache(wl, seed=seed, device=dev, lens=lens) if in_place else cache
        d, d2 = parity.make_desc(cache), parity.make_desc(twin)
        qc = cache.query_center.reshape(-1, wl.head_dim).to(dev).contiguous()
        w = tri.fold_weights(qc, wl.theta, wl.offsets)
        B = wl.budget
        assert d.units * tri.score_row_stride(d) <= 4 * 1024 * 1024

        def outputs():
            ko = vo = None
            if not in_place:
                ko = torch.zeros((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=dev)
                vo = torch.zeros((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=dev)
            return (torch.full((d.units, B), -1, dtype=torch.int32, device=dev),
                    torch.full((d.units,), -1, dtype=torch.int32, device=dev), ko, vo)

        kept, cnt, ko, vo = outputs()
        ws = torch.empty(tri.workspace_size(d, B), dtype=torch.uint8, device=dev)
        tri.compress(d, w, B, mode, kept, cnt, ko, vo, ws)
        kept2, cnt2, ko2, vo2 = outputs()
        n0 = tri.kernel_launches()
        _call_noalloc(fn, tri, d2, w, B, mode, kept2, cnt2, ko2, vo2)
        assert tri.kernel_launches() - n0 == launches
        assert tri.read_device_status() == 0
        torch.cuda.synchronize()
        assert torch.equal(cnt2, cnt)
        valid = torch.arange(B, device=dev)[None, :] < cnt[:, None]
        assert torch.equal(torch.where(valid, kept2, 0), torch.where(valid, kept, 0))
        if in_place:
            assert torch.equal(twin.k.view(torch.int16), cache.k.view(torch.int16))
            assert torch.equal(twin.v.view(torch.int16), cache.v.view(torch.int16))
        else:
            v3 = valid[:, :, None]
            assert torch.equal(torch.where(v3, ko2.view(torch.int16), 0), torch.where(v3, ko.view(torch.int16), 0))
            assert torch.equal(torch.where(v3, vo2.view(torch.int16), 0), torch.where(v3, vo.view(torch.int16), 0))


def test_noalloc_rejects_requests_beyond_its_scratch():
    import rope_aware_key_b200 as tri
    fn = _noalloc(tri.lib())
    dev = torch.device("cuda:0")
    k = torch.empty((1, 8, 1, 600000, 128), dtype=torch.bfloat16, device=dev)   # 4.8M scores > 4M
    d = tri.desc_contig(k, k)
    w = torch.zeros((8, 128), dtype=torch.float32, device=dev)
    kept = torch.empty((8, 16), dtype=torch.int32, device=dev)
    cnt = torch.empty((8,), dtype=torch.int32, device=dev)
    out = torch.empty((8, 16, 128), dtype=torch.bfloat16, device=dev)
    n0 = tri.kernel_launches()
    st = fn(d.ref, ctypes.c_void_p(w.data_ptr()), 16, tri.COMPACT_OUT_OF_PLACE, ctypes.c_void_p(kept.data_ptr()),
            ctypes.c_void_p(cnt.data_ptr()), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 3                       # TRI_ERR_WORKSPACE, nothing launched
    assert tri.kernel_launches() == n0
