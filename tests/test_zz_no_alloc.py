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


def test_noalloc_matches_compress_on_two_calls():
    import rope_aware_key_b200 as tri
    lib = tri.lib()
    fn = _noalloc(lib)
    dev = torch.device("cuda:0")
    # first call: a full 8-head layer; second call: a smaller ragged cache,
    # which must not be affected by the scores the first call left behind
    cases = [
        (gen.WORKLOADS["qwen3_layer"], None, 1),
        (gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=4, batch=3, budget=300), [900, 4000, 77], 2),
    ]
    for wl, lens, seed in cases:
        cache = gen.make_cache(wl, seed=seed, device=dev, lens=lens)
        d = parity.make_desc(cache)
        qc = cache.query_center.reshape(-1, wl.head_dim).to(dev).contiguous()
        w = tri.fold_weights(qc, wl.theta, wl.offsets)
        B = wl.budget
        assert d.units * tri.score_row_stride(d) <= 4 * 1024 * 1024

        def outputs():
            return (torch.full((d.units, B), -1, dtype=torch.int32, device=dev),
                    torch.full((d.units,), -1, dtype=torch.int32, device=dev),
                    torch.zeros((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=dev),
                    torch.zeros((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=dev))

        kept, cnt, ko, vo = outputs()
        tri.compress(d, w, B, tri.COMPACT_OUT_OF_PLACE, kept, cnt, ko, vo)
        kept2, cnt2, ko2, vo2 = outputs()
        st = fn(d.ref, ctypes.c_void_p(w.data_ptr()), B, tri.COMPACT_OUT_OF_PLACE,
                ctypes.c_void_p(kept2.data_ptr()), ctypes.c_void_p(cnt2.data_ptr()),
                ctypes.c_void_p(ko2.data_ptr()), ctypes.c_void_p(vo2.data_ptr()),
                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, tri.TriError(st, "tri_compress_noalloc")
        assert tri.read_device_status() == 0
        torch.cuda.synchronize()
        assert torch.equal(cnt2, cnt)
        valid = torch.arange(B, device=dev)[None, :] < cnt[:, None]
        assert torch.equal(torch.where(valid, kept2, 0), torch.where(valid, kept, 0))
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
