"""The max-over-offsets score (tensor-core kernel) against the oracle's
literal per-offset maximum, on the same seeded caches."""
import gc

import numpy as np
import pytest
import torch

import gen
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GEO17 = [float(2 ** e) for e in range(17)]


@pytest.fixture(autouse=True)
def _cleanup():
    yield
    gc.collect()
    if torch.cuda.is_available():
        torch.cuda.empty_cache()


def run_max(cache, offsets, delta0=0.0, pairing=0):
    import rope_aware_key_b200 as tri
    wl = cache.wl
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = tri.fold_offset_weights(qc, wl.theta, offsets, delta0, pairing)
    d = parity.make_desc(cache)
    scores = torch.full((d.units, tri.score_row_stride(d)), float("nan"), device=DEV)
    tri.score_keys_max(d, w, scores)
    status = tri.read_device_status()
    torch.cuda.synchronize()
    return w, scores, status


def check_offset_weights(w, cache, offsets, delta0, pairing):
    wl = cache.wl
    q = cache.query_center.reshape(-1, wl.head_dim)
    got = w.cpu().numpy().astype(np.float64)
    for t, dl in enumerate(offsets):
        ref = oracle.fold_w(q, wl.theta, [dl], delta0, pairing)
        err = np.abs(got[:, t] - ref)
        assert np.all(err <= 2.0 ** -23 * np.abs(ref) + 1e-12 * np.abs(ref).max()), t
    return got


def check_unit_max(cache, scores, w64, l, h, b, offsets, delta0, pairing, subset=None):
    """|s_gpu - s_ref| <= 1e-4 * max_t sum_j |w_t[j] k[j]| per key."""
    wl = cache.wl
    u = parity.unit_id(wl, l, h, b)
    n = cache.lens[b]
    keys = parity.bits16(gen.unit_rows(cache, cache.k, l, h, b))
    s = scores[u, :n].cpu().numpy().astype(np.float64)
    if subset:
        idx = np.linspace(0, n - 1, num=min(n, subset)).astype(np.int64)
        keys, s = keys[idx], s[idx]
    ref = oracle.score_max_literal(keys, cache.query_center[l, h].numpy(), wl.theta, offsets, delta0, pairing)
    lh = l * wl.num_kv_heads + h
    scale = np.max(np.stack([oracle.abs_dot(keys, w64[lh, t]) for t in range(len(offsets))]), axis=0)
    bad = np.flatnonzero(np.abs(s - ref) > parity.SCORE_TOL * scale)
    assert bad.size == 0, (u, bad[:5], s[bad[:5]], ref[bad[:5]])
    return float(np.max(np.abs(s - ref) / scale)) if n else 0.0


@pytest.mark.parametrize("n_off,pairing,delta0", [(17, 0, 0.0), (1, 0, 0.0), (5, 1, 3.0), (33, 0, 0.0), (64, 0, 100.0)])
def test_score_max_contig(n_off, pairing, delta0):
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=3, batch=2, seq_len=1000, theta=1e6)
    cache = gen.make_cache(wl, seed=21, device=DEV, with_values=False)
    offsets = GEO17[:n_off] if n_off <= 17 else [float(1 + 37 * i) for i in range(n_off)]
    w, scores, status = run_max(cache, offsets, delta0, pairing)
    assert status == 0
    w64 = check_offset_weights(w, cache, offsets, delta0, pairing)
    worst = 0.0
    for l in range(wl.num_layers):
        for h in range(wl.num_kv_heads):
            for b in range(wl.batch):
                worst = max(worst, check_unit_max(cache, scores, w64, l, h, b, offsets, delta0, pairing))
    assert worst < 1e-5
    assert torch.isnan(scores[:, 1000:]).all()          # row padding untouched


def test_score_max_ragged_edges():
    wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=7)
    cache = gen.make_cache(wl, seed=22, device=DEV, with_values=False, lens=[1, 127, 128, 129, 300, 0, 2049])
    w, scores, status = run_max(cache, GEO17)
    assert status == 0
    w64 = check_offset_weights(w, cache, GEO17, 0.0, 0)
    for l in range(2):
        for h in range(2):
            for b in range(7):
                check_unit_max(cache, scores, w64, l, h, b, GEO17, 0.0, 0)


@pytest.mark.parametrize("H,bs,n_off", [
    (4, 16, 17), (1, 128, 17), (2, 32, 17), (4, 4, 17), (8, 2, 16), (8, 16, 5), (2, 64, 64),  # whole pages
    (8, 1, 16), (2, 4, 17),                              # a page of all heads is one 8-row swizzle atom
    (8, 8, 17), (8, 16, 33), (4, 32, 64),                                                     # one head
])
def test_score_max_paged(H, bs, n_off):
    """Paged pools.  When every head's weights fit one MMA (H x n_cols <= 128)
    a tile is whole pages of all heads, one 2-box load per page; otherwise 128
    keys of one head, one 2-box load per page of that head."""
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=H, batch=4, block_size=bs,
                    spare_blocks_per_seq=1)
    cache = gen.make_cache(wl, seed=24 + H + bs + n_off, device=DEV, with_values=False, lens=[1, 127, 300, 1000])
    offsets = GEO17[:n_off] if n_off <= 17 else [float(1 + 37 * i) for i in range(n_off)]
    w, scores, status = run_max(cache, offsets)
    assert status == 0
    w64 = check_offset_weights(w, cache, offsets, 0.0, 0)
    for l in range(wl.num_layers):
        for h in range(H):
            for b in range(wl.batch):
                check_unit_max(cache, scores, w64, l, h, b, offsets, 0.0, 0)
    assert torch.isnan(scores[:, 1000:]).all()          # row padding untouched


@pytest.mark.parametrize("H,bs", [(4, 16), (1, 8), (8, 8)])    # whole pages x2, one head
def test_score_max_paged_empty_sequences(H, bs):
    """Sequences without keys among others: the tile walk steps past them."""
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=H, batch=6, block_size=bs,
                    spare_blocks_per_seq=1)
    lens = [0, 300, 0, 0, 17, 129]
    cache = gen.make_cache(wl, seed=40 + H + bs, device=DEV, with_values=False, lens=lens)
    w, scores, status = run_max(cache, GEO17)
    assert status == 0
    w64 = check_offset_weights(w, cache, GEO17, 0.0, 0)
    for l in range(wl.num_layers):
        for h in range(H):
            for b in range(wl.batch):
                check_unit_max(cache, scores, w64, l, h, b, GEO17, 0.0, 0)
    for b, n in enumerate(lens):                                  # nothing past each row's keys
        for l in range(wl.num_layers):
            for h in range(H):
                assert torch.isnan(scores[parity.unit_id(wl, l, h, b), n:]).all()


@pytest.mark.parametrize("H", [4, 8])                      # whole-page tiles, one-head tiles
def test_score_max_paged_bad_page_is_flagged_not_fatal(H):
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=1, num_kv_heads=H, batch=2, spare_blocks_per_seq=0)
    cache = gen.make_cache(wl, seed=29, device=DEV, with_values=False, lens=[200, 200])
    nb = cache.k.shape[1]
    cache.block_table[1, 3] = nb + 1000                     # tokens 48..63 of sequence 1: out of the pool
    w, scores, status = run_max(cache, GEO17)
    assert status & tri.DEVFLAG_BAD_PAGE
    tri.read_device_status(clear=True)
    assert tri.read_device_status() == 0
    w64 = check_offset_weights(w, cache, GEO17, 0.0, 0)
    for h in range(H):
        check_unit_max(cache, scores, w64, 0, h, 0, GEO17, 0.0, 0)        # the intact sequence is right
        u = parity.unit_id(wl, 0, h, 1)
        assert torch.isnan(scores[u, 48:64]).all()                     # the bad page's keys are not written
        assert not torch.isnan(scores[u, :48]).any() and not torch.isnan(scores[u, 64:200]).any()


def test_score_max_selects_like_the_oracle():
    """The kept set under the max score, through the same selection kernel."""
    import rope_aware_key_b200 as tri
    wl = gen.WORKLOADS["tiny"]
    cache = gen.make_cache(wl, seed=23, device=DEV)
    w, scores, status = run_max(cache, GEO17)
    d = parity.make_desc(cache)
    kept, cnt = tri.select_topk(d, scores, 512)
    torch.cuda.synchronize()
    s = scores[0, :4096].cpu().numpy()
    np.testing.assert_array_equal(kept[0].cpu().numpy(), oracle.select(s, 512))


def test_score_max_full_qwen3_sampled():
    """The 36 x 8 x 32768 cache, sampled units (every CTA crosses head boundaries)."""
    wl = gen.WORKLOADS["qwen3_full"]
    cache = gen.make_cache(wl, seed=0, device=DEV, with_values=False)
    w, scores, status = run_max(cache, GEO17)
    assert status == 0
    w64 = check_offset_weights(w, cache, GEO17, 0.0, 0)
    for (l, h) in [(0, 0), (17, 5), (35, 7)]:
        check_unit_max(cache, scores, w64, l, h, 0, GEO17, 0.0, 0, subset=2048)
    # every key of every unit was written
    assert not torch.isnan(scores).any()


def test_score_max_paged_full_steady_rows_sampled():
    """Config 5's steady-round rows as the bench scores them (28 layers x 4 KV
    heads x 64 sequences x 2176 keys in 16-token pages, whole-page tiles):
    sampled units against the oracle, and every key of every unit written."""
    wl = gen.WORKLOADS["qwen25_paged"]
    cache = gen.make_cache(wl, seed=5, device=DEV, with_values=False, lens=[2176] * wl.batch)
    w, scores, status = run_max(cache, GEO17)
    assert status == 0
    w64 = check_offset_weights(w, cache, GEO17, 0.0, 0)
    for (l, h, b) in [(0, 0, 0), (13, 2, 37), (27, 3, 63)]:
        check_unit_max(cache, scores, w64, l, h, b, GEO17, 0.0, 0, subset=1024)
    assert not torch.isnan(scores[:, :2176]).any()


def _max_calls(tri, d, w, B, mode, units, one_call):
    kept = torch.full((units, B), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((units,), -1, dtype=torch.int32, device=DEV)
    ko = vo = None
    if mode == tri.COMPACT_OUT_OF_PLACE:
        ko = torch.zeros((units, B, 128), dtype=torch.bfloat16, device=DEV)
        vo = torch.zeros_like(ko)
    if one_call:
        tri.compress_max(d, w, B, mode, kept, cnt, ko, vo)
    else:
        sc = tri.score_keys_max(d, w)
        tri.select_topk(d, sc, B, kept, cnt)
        tri.compact_kv(d, kept, cnt, B, mode, ko, vo)
    assert tri.read_device_status(clear=True) == 0
    return kept, cnt, ko, vo


@pytest.mark.parametrize("case", ["contig", "ragged", "paged_out_of_place", "paged_in_place", "paged_in_place_long"])
def test_compress_max_equals_the_three_calls(case):
    """tri_compress_max: the max scorer, then the selection (in place on short
    rows with the hole fill in the same warp) and the compaction, bit for bit
    the same as tri_score_keys_max + tri_select_topk + tri_compact_kv."""
    import rope_aware_key_b200 as tri
    mode = tri.COMPACT_OUT_OF_PLACE
    lens = None
    if case == "contig":
        wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=4, seq_len=4096, budget=700)
    elif case == "ragged":
        wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=5, budget=300)
        lens = [900, 5000, 77, 0, 301]
    elif case == "paged_out_of_place":
        wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, batch=4, budget=500, spare_blocks_per_seq=1)
        lens = [2176, 300, 0, 1999]
    else:
        mode = tri.COMPACT_IN_PLACE_HOLEFILL
        wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, batch=8, spare_blocks_per_seq=1)
        # B + 128 keys per row (the fill runs in the selection), or rows that move more than 512
        lens = [2176] * 8 if case == "paged_in_place" else [3000, 2176, 2047, 2900, 2600, 2048, 0, 3100]
    res = []
    for one_call in (True, False):
        cache = gen.make_cache(wl, seed=71, device=DEV, lens=lens)
        d = parity.make_desc(cache)
        qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
        w = tri.fold_offset_weights(qc, wl.theta, GEO17)
        out = _max_calls(tri, d, w, wl.budget, mode, d.units, one_call)
        torch.cuda.synchronize()
        res.append((out, cache))
    (a, ca), (b, cb) = res
    assert torch.equal(a[1], b[1])
    valid = torch.arange(wl.budget, device=DEV)[None, :] < a[1][:, None]
    assert torch.equal(torch.where(valid, a[0], 0), torch.where(valid, b[0], 0))
    if mode == tri.COMPACT_OUT_OF_PLACE:
        v3 = valid[:, :, None]
        for x, y in ((a[2], b[2]), (a[3], b[3])):
            assert torch.equal(torch.where(v3, x.view(torch.int16), 0), torch.where(v3, y.view(torch.int16), 0))
    else:                                   # the pools after the in-place fills
        assert torch.equal(ca.k.view(torch.int16), cb.k.view(torch.int16))
        assert torch.equal(ca.v.view(torch.int16), cb.v.view(torch.int16))


@pytest.mark.parametrize("group", [2, 4, 8])
def test_gqa_group_aggregation(group):
    """Grouped-query attention: several query heads share a KV head.  The
    pages leave their aggregation open; the two plain readings run on the
    existing calls.  Max over the group's query heads: each head's offset
    average folded on its own, then the max scorer over the group's weight
    vectors.  Mean over the group: the fold is linear in the center, so it is
    the folded score of the mean center."""
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=2, seq_len=900, theta=1e6)
    cache = gen.make_cache(wl, seed=81, device=DEV, with_values=False)
    rng = np.random.default_rng(81)
    LH = wl.num_layers * wl.num_kv_heads
    centers = rng.standard_normal((LH, group, 128)).astype(np.float32)      # one center per query head
    cd = torch.from_numpy(centers).to(DEV).reshape(LH * group, 128).contiguous()
    w_group = tri.fold_weights(cd, wl.theta, wl.offsets).reshape(LH, group, 128).contiguous()
    d = parity.make_desc(cache)
    s_max = torch.full((d.units, tri.score_row_stride(d)), float("nan"), device=DEV)
    tri.score_keys_max(d, w_group, s_max)
    mean_c = torch.from_numpy(centers.mean(axis=1)).to(DEV).contiguous()
    w_mean = tri.fold_weights(mean_c, wl.theta, wl.offsets)
    s_mean = tri.score_keys(d, w_mean)
    assert tri.read_device_status() == 0
    torch.cuda.synchronize()
    for l in range(wl.num_layers):
        for h in range(wl.num_kv_heads):
            lh = l * wl.num_kv_heads + h
            u = parity.unit_id(wl, l, h, 0)
            keys = parity.bits16(gen.unit_rows(cache, cache.k, l, h, 0))
            per_head = np.stack([oracle.score_literal(keys, centers[lh, i], wl.theta, wl.offsets) for i in range(group)])
            w64 = np.stack([oracle.fold_w(centers[lh, i][None, :], wl.theta, wl.offsets)[0] for i in range(group)])
            scale = np.max(np.stack([oracle.abs_dot(keys, w64[i]) for i in range(group)]), axis=0)
            got = s_max[u, :900].cpu().numpy().astype(np.float64)
            assert np.all(np.abs(got - per_head.max(axis=0)) <= parity.SCORE_TOL * scale)
            got_mean = s_mean[u, :900].cpu().numpy().astype(np.float64)
            wm = oracle.fold_w(centers[lh].mean(axis=0)[None, :].astype(np.float32), wl.theta, wl.offsets)[0]
            assert np.all(np.abs(got_mean - per_head.mean(axis=0)) <= parity.SCORE_TOL * oracle.abs_dot(keys, wm)
                          + 1e-9 * scale)
