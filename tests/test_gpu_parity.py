"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small cases compare every key of every unit with the oracle's literal
per-offset average; the full-size workloads run in the launch configuration
the bench times (fold, then the fused score -> select -> compact call) and
compare sampled units key by key, plus properties on every unit.
"""
import gc

import numpy as np
import pytest
import torch

import gen
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cleanup():
    yield
    gc.collect()
    if torch.cuda.is_available():
        torch.cuda.empty_cache()


def tri():
    import rope_aware_key_b200 as t
    return t


def check_every_unit(cache, res, pairing=0, delta0=None, literal=True, before=None, after=None):
    w64 = parity.check_fold(res, cache, pairing, delta0)
    wl = cache.wl
    reports = []
    for l in range(wl.num_layers):
        for h in range(wl.num_kv_heads):
            for b in range(wl.batch):
                kw = {}
                if before is not None:
                    kw = dict(before_k=before[(l, h, b)][0], before_v=before[(l, h, b)][1],
                              after_k=after[(l, h, b)][0], after_v=after[(l, h, b)][1])
                reports.append(parity.check_unit(cache, res, l, h, b, w64[l * wl.num_kv_heads + h],
                                                 literal=literal, pairing=pairing, delta0=delta0, **kw))
    parity.check_all_units_properties(cache, res)
    assert res.status == 0
    return reports


def snapshot(cache, units):
    out = {}
    for (l, h, b) in units:
        out[(l, h, b)] = (parity.bits16(gen.unit_rows(cache, cache.k, l, h, b)),
                          parity.bits16(gen.unit_rows(cache, cache.v, l, h, b)))
    return out


def all_units(wl):
    return [(l, h, b) for l in range(wl.num_layers) for h in range(wl.num_kv_heads) for b in range(wl.batch)]


# ------------------------------------------------------------------ small, every key

def test_tiny_single_head():
    cache = gen.make_cache(gen.WORKLOADS["tiny"], seed=0, device=DEV)
    res = parity.run_gpu(cache)
    reps = check_every_unit(cache, res)
    assert reps[0].max_err_over_l1 < 1e-5


def test_qwen3_layer_8x32768():
    cache = gen.make_cache(gen.WORKLOADS["qwen3_layer"], seed=0, device=DEV)
    res = parity.run_gpu(cache, fused=True)
    check_every_unit(cache, res)


@pytest.mark.parametrize("pairing,delta0", [(0, 0.0), (1, 5.0), (0, 1234.5)])
def test_contig_batch_ragged_tail(pairing, delta0):
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=3, batch=3, seq_len=1000, budget=100,
                    theta=1e6)
    cache = gen.make_cache(wl, seed=3, device=DEV)
    res = parity.run_gpu(cache, pairing=pairing, delta0=delta0)
    check_every_unit(cache, res, pairing=pairing, delta0=delta0)


def test_ragged_edge_lengths():
    wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=7, budget=128)
    lens = [1, 127, 128, 129, 300, 0, 2049]
    cache = gen.make_cache(wl, seed=5, device=DEV, lens=lens)
    for fused in (False, True):
        res = parity.run_gpu(cache, fused=fused)
        check_every_unit(cache, res)


@pytest.mark.parametrize("H", [1, 2, 4, 8])
def test_paged_out_of_place(H):
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=H, batch=5, budget=64,
                    spare_blocks_per_seq=1)
    cache = gen.make_cache(wl, seed=H, device=DEV, lens=[5, 16, 17, 300, 1000])
    res = parity.run_gpu(cache, mode=tri().COMPACT_OUT_OF_PLACE)
    check_every_unit(cache, res)


@pytest.mark.parametrize("H,fused", [(4, False), (8, True), (1, True)])
def test_paged_in_place_holefill(H, fused):
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=H, batch=5, budget=64,
                    spare_blocks_per_seq=1)
    cache = gen.make_cache(wl, seed=10 + H, device=DEV, lens=[5, 64, 65, 300, 1000])
    units = all_units(wl)
    before = snapshot(cache, units)
    res = parity.run_gpu(cache, mode=tri().COMPACT_IN_PLACE_HOLEFILL, fused=fused)
    after = snapshot(cache, units)
    check_every_unit(cache, res, before=before, after=after)


def test_contig_in_place_holefill():
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=2, seq_len=777, budget=200)
    cache = gen.make_cache(wl, seed=4, device=DEV)
    units = all_units(wl)
    before = snapshot(cache, units)
    res = parity.run_gpu(cache, mode=tri().COMPACT_IN_PLACE_HOLEFILL)
    after = snapshot(cache, units)
    check_every_unit(cache, res, before=before, after=after)


# Rows of at most 4096 keys are selected by one warp each, longer rows by one
# CTA each: the selection edge cases below run at a length of each kind.
WARP_ROW, CTA_ROW = 1000, 5000


@pytest.mark.parametrize("n", [WARP_ROW, CTA_ROW])
@pytest.mark.parametrize("budget", ["1", "2", "n-1", "n", "n+5"])
def test_budget_edges(n, budget):
    B = {"1": 1, "2": 2, "n-1": n - 1, "n": n, "n+5": n + 5}[budget]
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=1, seq_len=n, budget=B)
    cache = gen.make_cache(wl, seed=6, device=DEV)
    res = parity.run_gpu(cache)
    check_every_unit(cache, res)


@pytest.mark.parametrize("n", [3000, 6000])
def test_exact_ties_go_to_lower_index(n):
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=1, batch=1, seq_len=n, budget=700 * n // 3000)
    cache = gen.make_cache(wl, seed=7, device=DEV)
    # 37 distinct rows repeated: every score appears n / 37 times, exactly
    base = cache.k[0, 0, 0, :37].clone()
    cache.k[0, 0, 0] = base.repeat(n // 37 + 1, 1)[:n]
    res = parity.run_gpu(cache)
    check_every_unit(cache, res)
    s = res.scores[0, :n].cpu().numpy()
    kept = res.kept[0].cpu().numpy()
    t = s[kept].min()
    eq = np.flatnonzero(s == t)
    kept_eq = np.intersect1d(eq, kept)
    assert len(kept_eq) < len(eq) and np.array_equal(kept_eq, eq[: len(kept_eq)])


@pytest.mark.parametrize("n", [4096, 4100])
def test_all_scores_equal(n):
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=1, batch=1, seq_len=n, budget=333)
    cache = gen.make_cache(wl, seed=8, device=DEV)
    cache.k[0, 0, 0] = cache.k[0, 0, 0, :1].expand(n, -1)
    res = parity.run_gpu(cache)
    check_every_unit(cache, res)
    assert np.array_equal(res.kept[0].cpu().numpy(), np.arange(333))


def test_long_rows_select_without_shared_cache():
    """Rows longer than the shared-memory key cache take the uncached path."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=1, seq_len=50001, budget=3000,
                    theta=5e5)
    cache = gen.make_cache(wl, seed=15, device=DEV)
    res = parity.run_gpu(cache)
    check_every_unit(cache, res, literal=False)


@pytest.mark.parametrize("n,B", [(10000, 4100), (4096, 1700)])
def test_heavy_duplicates_overflow_path(n, B):
    """Three distinct scores: the threshold's bin holds more keys than the
    candidate list, so the selection takes its fallback path."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=1, seq_len=n, budget=B)
    cache = gen.make_cache(wl, seed=13, device=DEV)
    for h in range(2):
        base = cache.k[0, h, 0, :3].clone()
        cache.k[0, h, 0] = base.repeat(n // 3 + 1, 1)[:n]
    res = parity.run_gpu(cache)
    check_every_unit(cache, res)


@pytest.mark.parametrize("n", [3000, 5000])
def test_single_finite_value_with_infinities(n):
    """One finite score value plus +/-inf keys: no finite range to bin."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=1, batch=1, seq_len=n, budget=1500)
    cache = gen.make_cache(wl, seed=14, device=DEV)
    k = cache.k[0, 0, 0]
    k[:] = k[:1].clone()
    k[100, :] = float("inf")
    k[200, :] = float("-inf")
    res = parity.run_gpu(cache)
    s = res.scores[0, :n].cpu().numpy()
    kept = res.kept[0, :1500].cpu().numpy()
    np.testing.assert_array_equal(kept, oracle.select(s, 1500))
    assert res.status == 0


@pytest.mark.parametrize("n", [600, 4600])
def test_nonfinite_keys_rank_lowest(n):
    """NaN scores rank lowest; +/-inf keys give +/-inf or NaN scores."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=1, batch=1, seq_len=n, budget=n - 10)
    cache = gen.make_cache(wl, seed=9, device=DEV)
    k = cache.k[0, 0, 0]
    k[10] = float("nan")
    k[20, 5] = float("inf")
    k[30, 7] = float("-inf")
    k[40] = 0.0
    res = parity.run_gpu(cache)
    s = res.scores[0, :n].cpu().numpy()
    assert np.isnan(s[10])
    kept = res.kept[0, :n - 10].cpu().numpy()
    np.testing.assert_array_equal(kept, oracle.select(s, n - 10))
    assert 10 not in set(kept.tolist())
    # finite keys: scores within tolerance of the oracle
    w64 = parity.check_fold(res, cache)
    keys = parity.bits16(k)
    fin = np.all(np.isfinite(k.float().cpu().numpy()), axis=1)
    ref = oracle.score_literal(keys[fin], cache.query_center[0, 0].numpy(), wl.theta, wl.offsets)
    parity.check_scores(keys[fin], s[fin], ref, w64[0])


@pytest.mark.parametrize("n,B,nans", [(1000, 900, 200), (4000, 3990, 64), (5000, 4900, 300)])
def test_fewer_numbers_than_budget_keeps_lowest_nans(n, B, nans):
    """More NaN scores than n - B: the threshold is NaN itself, and the
    lowest-index NaN keys fill the budget."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=1, batch=1, seq_len=n, budget=B)
    cache = gen.make_cache(wl, seed=17, device=DEV)
    rng = np.random.default_rng(n)
    bad = np.sort(rng.choice(n, size=nans, replace=False))
    cache.k[0, 0, 0, torch.as_tensor(bad, device=DEV)] = float("nan")
    res = parity.run_gpu(cache)
    s = res.scores[0, :n].cpu().numpy()
    assert np.isnan(s[bad]).all()
    kept = res.kept[0, :B].cpu().numpy()
    np.testing.assert_array_equal(kept, oracle.select(s, B))
    assert int(res.kept_count[0]) == B


def test_steady_round_shape_every_unit():
    """The shape of a paged cache re-compressed every 128 generated tokens:
    rows of B + 128 keys (and shorter ones), 16-token pages of 4 KV heads,
    compacted in place; every key of every unit against the oracle."""
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=4, batch=6, budget=2048,
                    spare_blocks_per_seq=1)
    cache = gen.make_cache(wl, seed=18, device=DEV, lens=[2176, 2176, 2048, 2175, 2049, 4096])
    units = all_units(wl)
    before = snapshot(cache, units)
    res = parity.run_gpu(cache, mode=tri().COMPACT_IN_PLACE_HOLEFILL)
    after = snapshot(cache, units)
    check_every_unit(cache, res, literal=False, before=before, after=after)


@pytest.mark.parametrize("lens,B", [([2176, 2176, 2048, 2175, 2049, 2560], 2048),
                                    ([4096, 3700, 4000, 100, 3601], 3600)])
def test_compress_in_place_fills_holes_in_the_selection(lens, B):
    """tri_compress in place on rows that move at most 512 keys: one warp per
    row selects and then fills the row's holes, from its evicted list (rows
    that evict few keys) or from its kept list (the others).  Three launches
    (fold, score, the selection with the fill); every unit against the
    oracle, K and V before and after."""
    t = tri()
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=4, batch=len(lens), budget=B,
                    spare_blocks_per_seq=1)
    cache = gen.make_cache(wl, seed=21 + B, device=DEV, lens=lens)
    units = all_units(wl)
    before = snapshot(cache, units)
    n0 = t.kernel_launches()
    res = parity.run_gpu(cache, mode=t.COMPACT_IN_PLACE_HOLEFILL, fused=True)
    assert t.kernel_launches() - n0 == 3
    after = snapshot(cache, units)
    check_every_unit(cache, res, literal=False, before=before, after=after)


@pytest.mark.parametrize("H,bs,B,lens", [
    (8, 12, 2000, [2001, 2127, 2128, 2129, 2512, 1999]),   # pages of 12 tokens (no shift), B not a multiple of 32
    (1, 32, 1000, [1512, 1129, 1001, 700]),                 # tails of 1..512 rows: several 128-position chunks
    (2, 64, 3000, [3500, 3200, 3001, 3000]),
])
def test_compress_in_place_fill_page_shapes(H, bs, B, lens):
    """The selection's in-kernel fill on paged caches of other page sizes and
    head counts, tails that span several chunks and budgets that split a
    bitmap word; every unit against the oracle, K and V before and after."""
    t = tri()
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=H, batch=len(lens), budget=B,
                    block_size=bs, spare_blocks_per_seq=1)
    cache = gen.make_cache(wl, seed=40 + H + bs, device=DEV, lens=lens)
    units = all_units(wl)
    before = snapshot(cache, units)
    n0 = t.kernel_launches()
    res = parity.run_gpu(cache, mode=t.COMPACT_IN_PLACE_HOLEFILL, fused=True)
    assert t.kernel_launches() - n0 == 3                       # fold, score, the selection with the fill
    after = snapshot(cache, units)
    check_every_unit(cache, res, literal=False, before=before, after=after)


@pytest.mark.parametrize("dup", [1, 3])
def test_compress_in_place_fill_after_the_whole_row_search(dup):
    """Rows whose scores take one or three values: the selection's bracket
    check fails and the whole-row search decides; the fill in the same kernel
    then follows the kept list.  Contiguous cache, in place."""
    n, B = 2400, 2000
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=1, seq_len=n, budget=B)
    cache = gen.make_cache(wl, seed=22 + dup, device=DEV)
    for h in range(2):
        base = cache.k[0, h, 0, :dup].clone()
        cache.k[0, h, 0] = base.repeat(n // dup + 1, 1)[:n]
    units = all_units(wl)
    before = snapshot(cache, units)
    res = parity.run_gpu(cache, mode=tri().COMPACT_IN_PLACE_HOLEFILL, fused=True)
    after = snapshot(cache, units)
    check_every_unit(cache, res, before=before, after=after)


def test_in_place_budget_above_16384():
    """The hole fill has no budget limit of its own."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=1, seq_len=20000, budget=17000)
    cache = gen.make_cache(wl, seed=20, device=DEV)
    units = all_units(wl)
    before = snapshot(cache, units)
    res = parity.run_gpu(cache, mode=tri().COMPACT_IN_PLACE_HOLEFILL)
    after = snapshot(cache, units)
    check_every_unit(cache, res, literal=False, before=before, after=after)


def test_second_round_rows_crowd_at_the_threshold():
    """After one pruning event every row holds the survivors, which all sit
    just above the old threshold; 128 new tokens later the new threshold lies
    among them, in a crowded value range (the warp selection bins that range
    again).  Two events on a paged cache, every unit against the oracle."""
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, num_kv_heads=4, batch=3, budget=2048,
                    spare_blocks_per_seq=8)
    cache = gen.make_cache(wl, seed=19, device=DEV, lens=[20000, 32768, 9000])
    t = tri()
    parity.run_gpu(cache, mode=t.COMPACT_IN_PLACE_HOLEFILL)
    gen.release_tail_blocks(cache, [min(wl.budget, n) for n in cache.lens])
    gen.append_tokens(cache, 128, step=1)
    units = all_units(wl)
    before = snapshot(cache, units)
    res = parity.run_gpu(cache, mode=t.COMPACT_IN_PLACE_HOLEFILL)
    after = snapshot(cache, units)
    check_every_unit(cache, res, literal=False, before=before, after=after)


def test_score_row_padding():
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=1, num_kv_heads=2, batch=1, seq_len=513, budget=64)
    cache = gen.make_cache(wl, seed=11, device=DEV)
    res = parity.run_gpu(cache, max_seq_len=1001)
    assert res.scores.shape[1] == 1004
    assert torch.isnan(res.scores[:, 513:]).all()      # padding never written
    check_every_unit(cache, res)


def test_bad_page_is_flagged_not_fatal():
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=1, num_kv_heads=4, batch=2, budget=16,
                    spare_blocks_per_seq=0)
    cache = gen.make_cache(wl, seed=12, device=DEV, lens=[40, 40])
    nb = cache.k.shape[1]
    cache.block_table[1, 1] = nb + 1000            # out of the pool
    res = parity.run_gpu(cache)
    assert res.status & tri().DEVFLAG_BAD_PAGE
    # the intact sequence is still right
    w64 = parity.check_fold(res, cache)
    for h in range(4):
        parity.check_unit(cache, res, 0, h, 0, w64[h])
    assert tri().read_device_status() == 0           # cleared


def test_launch_count_and_status_clean():
    t = tri()
    cache = gen.make_cache(gen.WORKLOADS["tiny"], seed=0, device=DEV)
    n0 = t.kernel_launches()
    parity.run_gpu(cache, fused=True)
    assert t.kernel_launches() - n0 == 2            # fold, then one cluster kernel (one unit)
    n0 = t.kernel_launches()
    parity.run_gpu(cache, fused=False)
    assert t.kernel_launches() - n0 == 4            # fold, score, select, compact
    # a cache with more units than one wave of clusters takes the three kernels
    many = gen.make_cache(gen.scaled(gen.WORKLOADS["tiny"], num_layers=20, num_kv_heads=8, seq_len=300),
                          seed=0, device=DEV)
    n0 = t.kernel_launches()
    res = parity.run_gpu(many, fused=True)
    assert t.kernel_launches() - n0 == 4 and res.status == 0
    check_every_unit(many, res, literal=False)


# ------------------------------------------------------------------ full size, sampled

def sample_units(wl, k, seed):
    rng = np.random.default_rng(seed)
    units = {(0, 0, 0), (wl.num_layers - 1, wl.num_kv_heads - 1, wl.batch - 1)}
    while len(units) < k:
        units.add((int(rng.integers(wl.num_layers)), int(rng.integers(wl.num_kv_heads)),
                   int(rng.integers(wl.batch))))
    return sorted(units)


def check_sampled(cache, res, units, before=None, after=None, literal_subset=512):
    w64 = parity.check_fold(res, cache)
    H = cache.wl.num_kv_heads
    for (l, h, b) in units:
        kw = {}
        if before is not None:
            kw = dict(before_k=before[(l, h, b)][0], before_v=before[(l, h, b)][1],
                      after_k=after[(l, h, b)][0], after_v=after[(l, h, b)][1])
        parity.check_unit(cache, res, l, h, b, w64[l * H + h], literal=False, literal_subset=literal_subset, **kw)
    parity.check_all_units_properties(cache, res)
    assert res.status == 0


def test_full_qwen3_36x8x32768():
    """The bench workload."""
    wl = gen.WORKLOADS["qwen3_full"]
    cache = gen.make_cache(wl, seed=0, device=DEV)
    res = parity.run_gpu(cache, fused=True)
    check_sampled(cache, res, sample_units(wl, 5, 1))


def test_full_qwen3_ragged_batch8():
    wl = gen.WORKLOADS["qwen3_ragged"]
    cache = gen.make_cache(wl, seed=0, device=DEV)
    res = parity.run_gpu(cache, fused=True)
    check_sampled(cache, res, sample_units(wl, 5, 2))


def test_full_llama3_long_uniform_schedule():
    wl = gen.WORKLOADS["llama3_long"]
    cache = gen.make_cache(wl, seed=0, device=DEV)
    res = parity.run_gpu(cache, fused=True)
    check_sampled(cache, res, sample_units(wl, 3, 3), literal_subset=256)


def test_full_paged_incremental_rounds():
    """Initial compression of the paged cache, then rounds of 128 appended
    tokens per sequence re-compressed in place down to B."""
    wl = gen.WORKLOADS["qwen25_paged"]
    cache = gen.make_cache(wl, seed=0, device=DEV)
    t = tri()
    for rnd in range(3):
        if rnd > 0:
            gen.append_tokens(cache, 128, step=rnd)
        units = sample_units(wl, 4, 10 + rnd)
        before = snapshot(cache, units)
        res = parity.run_gpu(cache, mode=t.COMPACT_IN_PLACE_HOLEFILL, fused=True)
        after = snapshot(cache, units)
        check_sampled(cache, res, units, before=before, after=after)
        gen.release_tail_blocks(cache, [min(wl.budget, n) for n in cache.lens])


def test_fold_follows_every_schedule_change():
    """The host keeps the factors of the last schedule: alternating schedules,
    offsets and kept distances must each give their own weights."""
    t = tri()
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_kv_heads=3)
    q = gen.make_cache(wl, seed=71, device=DEV, with_values=False).query_center.reshape(-1, 128)
    qd = q.to(DEV).contiguous()
    geo = [float(2 ** e) for e in range(17)]
    cases = [(1e4, geo, 0.0), (1e6, geo, 0.0), (1e6, geo, 7.0), (1e6, geo[:-1] + [65537.0], 0.0),
             (1e4, geo, 0.0), (5e5, [float(i) for i in range(1, 1025)], 0.0), (1e4, geo, 0.0)]
    for theta, offs, d0 in cases:
        for pairing in (0, 1):
            w = t.fold_weights(qd, theta, offs, d0, pairing).cpu().numpy().astype(np.float64)
            ref = oracle.fold_w(q, theta, offs, d0, pairing)
            err = np.abs(w - ref)
            assert np.all(err <= 2.0 ** -23 * np.abs(ref) + 1e-12 * np.abs(ref).max()), (theta, len(offs), d0)


def test_binding_refuses_short_or_mistyped_buffers():
    """A device buffer one row short, of the wrong dtype or strided is refused
    on the host, before any launch; the right sizes go through."""
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=2, seq_len=300, budget=64)
    cache = gen.make_cache(wl, seed=51, device=DEV)
    d = parity.make_desc(cache)
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = tri.fold_weights(qc, wl.theta, wl.offsets)
    stride = tri.score_row_stride(d)
    B = wl.budget
    launches = tri.kernel_launches()
    with pytest.raises(ValueError, match="w: need"):
        tri.score_keys(d, w[:-1])
    with pytest.raises(ValueError, match="scores: need"):
        tri.score_keys(d, w, torch.empty((d.units, stride - 4), device=DEV))
    with pytest.raises(ValueError, match="scores: need"):
        tri.score_keys(d, w, torch.empty((stride, d.units), device=DEV).t())
    scores = tri.score_keys(d, w)
    with pytest.raises(ValueError, match="kept: need"):
        tri.select_topk(d, scores, B, torch.empty((d.units, B - 1), dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError, match="kept_count: need"):
        tri.select_topk(d, scores, B, None, torch.empty((d.units,), dtype=torch.int64, device=DEV))
    kept, cnt = tri.select_topk(d, scores, B)
    short = torch.empty((d.units, B - 1, wl.head_dim), dtype=torch.bfloat16, device=DEV)
    full = torch.empty((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError, match="k_out: need"):
        tri.compact_kv(d, kept, cnt, B, tri.COMPACT_OUT_OF_PLACE, short, full)
    with pytest.raises(ValueError, match="v_out: need"):
        tri.compact_kv(d, kept, cnt, B, tri.COMPACT_OUT_OF_PLACE, full, full.float())
    with pytest.raises(ValueError, match="positions: need"):
        tri.score_keys_at_positions(d, w, wl.theta, [300], torch.zeros((d.units, stride - 4), dtype=torch.int32,
                                                                        device=DEV))
    with pytest.raises(ValueError, match="query_pos: need one position per sequence"):
        tri.score_keys_at_positions(d, w, wl.theta, [])
    assert tri.kernel_launches() == launches + 2          # the two calls that went through
    tri.compact_kv(d, kept, cnt, B, tri.COMPACT_OUT_OF_PLACE, full, torch.empty_like(full))
    assert tri.read_device_status() == 0
