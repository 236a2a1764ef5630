"""Failure detection on the device, without faulting the GPU.

Two test-only builds of the library's sources (never the product library):

* "hooks": every bounded wait gives up after 1 ms instead of about 2 s, and
  the producer of the folded scorer or of the max scorer can be told to leave
  one tile out -- no copy and no arrival on its barrier.  The consumers of that tile then wait in vain,
  give up, set TRI_DEVFLAG_TIMEOUT and leave the kernel; the producer's own
  waits end the same way, after it has waited for every copy it did issue,
  so no copy is in flight into an exiting CTA.  The host reads
  TRI_ERR_DEVICE_TIMEOUT, and the next call on the same device is clean and
  right.
* "checked": device-side invariants of the selection and compaction (kept
  counts, histogram totals, holes against movers).  On correct inputs the
  status stays clean and the results equal the product build's bit for bit;
  a kept count planted on the host (in range, so nothing is read out of
  bounds) is reported as TRI_DEVFLAG_INVARIANT.
"""
import ctypes

import numpy as np
import pytest
import torch

import gen
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _variant(name, monkeypatch):
    import rope_aware_key_b200 as tri
    from rope_aware_key_b200 import build as tri_build
    V = tri.load(tri_build.build_variant(name))
    tri.lib()                                    # the product build stays loaded beside it
    monkeypatch.setattr(tri, "_lib", V)          # the binding now calls the variant
    return tri, V


def _check_units(cache, res, units):
    w64 = parity.check_fold(res, cache)
    H = cache.wl.num_kv_heads
    for (l, h, b) in units:
        parity.check_unit(cache, res, l, h, b, w64[l * H + h], literal=False, literal_subset=128)


def test_bounded_wait_runs_out_then_recovers(monkeypatch):
    tri, V = _variant("hooks", monkeypatch)
    wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], seq_len=32768)       # 8 x 256 tiles of 128 keys
    cache = gen.make_cache(wl, seed=21, device=DEV)
    d = parity.make_desc(cache)
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = tri.fold_weights(qc, wl.theta, wl.offsets)
    assert tri.read_device_status() == 0
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    V.tri_test_skip_tile(sms + 4)                # the second tile of one CTA (grid <= 2 per SM, >= 148)
    try:
        scores = tri.score_keys(d, w)
        flags = ctypes.c_uint32(0)
        st = V.tri_read_device_status(tri._stream(None), ctypes.byref(flags), 1)
    finally:
        V.tri_test_skip_tile(-1)
    assert st == 6                               # TRI_ERR_DEVICE_TIMEOUT
    assert flags.value & tri.DEVFLAG_TIMEOUT
    assert scores.shape[0] == d.units
    # the same device, the next call: clean and right
    res = parity.run_gpu(cache)
    assert res.status == 0
    _check_units(cache, res, [(0, 0, 0), (0, 3, 0), (0, 7, 0)])
    parity.check_all_units_properties(cache, res)


@pytest.mark.parametrize("layout", ["contig", "paged"])
def test_max_scorer_wait_runs_out_then_recovers(layout, monkeypatch):
    """The tensor-core max scorer: its producer leaves one tile out; the MMA
    thread's wait gives up, the epilogue and the producer stop, the producer
    waits for the copies it did issue and the MMA thread for its last commit
    before the tensor memory is freed; the next call is clean and right."""
    from tests import test_gpu_score_max as tm
    tri, V = _variant("hooks", monkeypatch)
    if layout == "contig":
        wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], seq_len=32768)      # 2048 tiles, ~14 per CTA
        cache = gen.make_cache(wl, seed=31, device=DEV, with_values=False)
        skip = 20
    else:                                                                # whole-page tiles of 4 heads
        wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, batch=8, spare_blocks_per_seq=1)
        cache = gen.make_cache(wl, seed=32, device=DEV, with_values=False, lens=[2176] * 8)
        skip = 10
    d = parity.make_desc(cache)
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = tri.fold_offset_weights(qc, wl.theta, tm.GEO17)
    assert tri.read_device_status() == 0
    V.tri_test_skip_tile(skip)
    try:
        tri.score_keys_max(d, w)
        flags = ctypes.c_uint32(0)
        st = V.tri_read_device_status(tri._stream(None), ctypes.byref(flags), 1)
    finally:
        V.tri_test_skip_tile(-1)
    assert st == 6                               # TRI_ERR_DEVICE_TIMEOUT
    assert flags.value & tri.DEVFLAG_TIMEOUT
    # the same device, the next call: clean and right
    w2, scores, status = tm.run_max(cache, tm.GEO17)
    assert status == 0
    w64 = tm.check_offset_weights(w2, cache, tm.GEO17, 0.0, 0)
    H = wl.num_kv_heads
    for (l, h, b) in [(0, 0, 0), (wl.num_layers - 1, H - 1, wl.batch - 1)]:
        tm.check_unit_max(cache, scores, w64, l, h, b, tm.GEO17, 0.0, 0, subset=1024)
    assert not torch.isnan(scores[:, :max(cache.lens)]).any()


def _same(a, b):
    assert torch.equal(a.kept_count, b.kept_count)
    B = a.kept.shape[1]
    valid = torch.arange(B, device=a.kept.device)[None, :] < a.kept_count[:, None]
    assert torch.equal(torch.where(valid, a.kept, 0), torch.where(valid, b.kept, 0))
    if a.k_out is not None:
        v3 = valid[:, :, None]
        for x, y in ((a.k_out, b.k_out), (a.v_out, b.v_out)):
            assert torch.equal(torch.where(v3, x.view(torch.int16), 0), torch.where(v3, y.view(torch.int16), 0))


@pytest.mark.parametrize("case", ["tiny", "ragged_edges", "layer_fused", "paged_in_place", "long_rows"])
def test_checked_build_clean_and_identical(case, monkeypatch):
    import rope_aware_key_b200 as prod
    lens = None
    mode, fused = prod.COMPACT_OUT_OF_PLACE, False
    if case == "tiny":
        wl = gen.WORKLOADS["tiny"]
    elif case == "ragged_edges":
        wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=7, budget=128)
        lens = [1, 127, 128, 129, 300, 0, 2049]
    elif case == "layer_fused":
        wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], seq_len=8192)
        fused = True
    elif case == "paged_in_place":
        wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=4, batch=4, budget=2048,
                        spare_blocks_per_seq=1)
        lens = [2176, 2176, 9000, 100]
        mode = prod.COMPACT_IN_PLACE_HOLEFILL
    else:
        wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, seq_len=50001, budget=3000)
    ref_cache = gen.make_cache(wl, seed=31, device=DEV, lens=lens)
    ref = parity.run_gpu(ref_cache, mode=mode, fused=fused)           # product build
    assert ref.status == 0
    tri, _ = _variant("checked", monkeypatch)
    cache = gen.make_cache(wl, seed=31, device=DEV, lens=lens)
    units = [(0, 0, b) for b in range(wl.batch)]
    before = {u: (parity.bits16(gen.unit_rows(cache, cache.k, *u)), parity.bits16(gen.unit_rows(cache, cache.v, *u)))
              for u in units} if mode == prod.COMPACT_IN_PLACE_HOLEFILL else None
    res = parity.run_gpu(cache, mode=mode, fused=fused)
    assert res.status == 0, f"device status {res.status:#x}"
    _same(res, ref)
    w64 = parity.check_fold(res, cache)
    for (l, h, b) in units:
        kw = {}
        if before is not None:
            kw = dict(before_k=before[(l, h, b)][0], before_v=before[(l, h, b)][1],
                      after_k=parity.bits16(gen.unit_rows(cache, cache.k, l, h, b)),
                      after_v=parity.bits16(gen.unit_rows(cache, cache.v, l, h, b)))
        parity.check_unit(cache, res, l, h, b, w64[l * wl.num_kv_heads + h], literal=False, **kw)
    if mode == prod.COMPACT_IN_PLACE_HOLEFILL:
        assert torch.equal(cache.k.view(torch.int16), ref_cache.k.view(torch.int16))


def test_checked_build_reports_a_planted_kept_count(monkeypatch):
    tri, _ = _variant("checked", monkeypatch)
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, seq_len=1000, budget=100)
    cache = gen.make_cache(wl, seed=32, device=DEV)
    res = parity.run_gpu(cache)
    assert res.status == 0
    d = parity.make_desc(cache)
    cnt = res.kept_count.clone()
    cnt[1] -= 1                                  # one row fewer than the selection kept: still in range
    k_out, v_out = torch.zeros_like(res.k_out), torch.zeros_like(res.v_out)
    tri.compact_kv(d, res.kept, cnt, wl.budget, tri.COMPACT_OUT_OF_PLACE, k_out, v_out)
    assert tri.read_device_status() & tri.DEVFLAG_INVARIANT
    assert tri.read_device_status() == 0         # cleared by the read
    # the rows it did copy are the selection's
    assert torch.equal(k_out[0].view(torch.int16), res.k_out[0].view(torch.int16))
    n = int(cnt[1])
    assert torch.equal(k_out[1, :n].view(torch.int16), res.k_out[1, :n].view(torch.int16))
    assert not np.any(k_out[1, n:].float().cpu().numpy())
