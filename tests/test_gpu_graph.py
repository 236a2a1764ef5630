"""The step as the bench times it: fold, score, select and compact captured
once in a CUDA graph and replayed.  The graph must give, bit for bit, what
plain launches give, and a replay must read the cache's current contents
(the graph holds pointers, not data)."""
import gc

import pytest
import torch

import gen
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cleanup():
    yield
    gc.collect()
    if torch.cuda.is_available():
        torch.cuda.empty_cache()


def test_graph_replay_matches_plain_launches():
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["qwen3_8layers"], num_layers=2)
    cache = gen.make_cache(wl, seed=61, device=DEV)
    d = tri.desc_contig(cache.k, cache.v)
    qc = cache.query_center.reshape(-1, 128).to(DEV).contiguous()
    B = wl.budget
    w = torch.empty_like(qc)
    scores = torch.empty((d.units, tri.score_row_stride(d)), device=DEV)
    kept = torch.empty((d.units, B), dtype=torch.int32, device=DEV)
    cnt = torch.empty((d.units,), dtype=torch.int32, device=DEV)
    ko = torch.empty((d.units, B, 128), dtype=torch.bfloat16, device=DEV)
    vo = torch.empty_like(ko)

    def step():
        st = torch.cuda.current_stream()
        tri.fold_weights(qc, wl.theta, wl.offsets, wl.delta0, 0, out=w, stream=st)
        tri.score_keys(d, w, scores, stream=st)
        tri.select_topk(d, scores, B, kept, cnt, stream=st)
        tri.compact_kv(d, kept, cnt, B, tri.COMPACT_OUT_OF_PLACE, ko, vo, stream=st)

    step()
    torch.cuda.synchronize()
    plain = [x.clone() for x in (w, scores, kept, cnt, ko, vo)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    for x in (w, scores, kept, cnt, ko, vo):
        x.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(plain, (w, scores, kept, cnt, ko, vo)):
        assert torch.equal(a, b)
    # new cache contents in the same buffers: the replay sees them
    other = gen.make_cache(wl, seed=62, device=DEV)
    cache.k.copy_(other.k)
    cache.v.copy_(other.v)
    qc.copy_(other.query_center.reshape(-1, 128).to(DEV))
    graph.replay()
    torch.cuda.synchronize()
    replayed = [x.clone() for x in (w, scores, kept, cnt, ko, vo)]
    step()
    torch.cuda.synchronize()
    for a, b in zip(replayed, (w, scores, kept, cnt, ko, vo)):
        assert torch.equal(a, b)
    assert not torch.equal(replayed[2], plain[2])
    assert tri.read_device_status() == 0
    # and the replayed results are right (sampled units against the oracle)
    res = parity.GpuResult(w, scores, kept, cnt, ko, vo, 0, B, tri.COMPACT_OUT_OF_PLACE)
    other.k, other.v = cache.k, cache.v
    w64 = parity.check_fold(res, other)
    for (l, h) in [(0, 0), (1, 7)]:
        parity.check_unit(other, res, l, h, 0, w64[l * wl.num_kv_heads + h], literal_subset=512)
