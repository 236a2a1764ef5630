"""The single-kernel step (one thread-block cluster per unit: score, select,
compact) against the three-kernel path and the oracle.  Both paths score with
the same lanes in the same order, so their scores, kept indices and compacted
rows must be identical, bit for bit."""
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


def fold64(cache):
    wl = cache.wl
    return oracle.fold_w(cache.query_center.reshape(-1, wl.head_dim), wl.theta, wl.offsets, wl.delta0, 0)


def both_paths(cache, B):
    """(single kernel via tri_compress, three kernels via the separate calls)."""
    import rope_aware_key_b200 as tri
    fused = parity.run_gpu(cache, budget=B, fused=True)
    split = parity.run_gpu(cache, budget=B, fused=False)
    return fused, split


def assert_same(cache, fused, split, B):
    assert fused.status == 0 and split.status == 0
    units = fused.kept.shape[0]
    for u in range(units):
        b = u % cache.wl.batch
        n = cache.lens[b]
        m = min(B, n)
        np.testing.assert_array_equal(fused.scores[u, :n].cpu().numpy().view(np.uint32),
                                      split.scores[u, :n].cpu().numpy().view(np.uint32))
        assert int(fused.kept_count[u]) == m == int(split.kept_count[u])
        np.testing.assert_array_equal(fused.kept[u, :m].cpu().numpy(), split.kept[u, :m].cpu().numpy())
        assert torch.equal(fused.k_out[u, :m], split.k_out[u, :m])
        assert torch.equal(fused.v_out[u, :m], split.v_out[u, :m])


def test_single_kernel_step_8_units():
    """One layer of a Qwen3-shaped cache (8 KV heads x 8192 keys): 8 clusters."""
    wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], seq_len=8192)
    cache = gen.make_cache(wl, seed=51, device=DEV)
    fused, split = both_paths(cache, wl.budget)
    assert_same(cache, fused, split, wl.budget)
    # and against the oracle on two units (scores, exact selection on the GPU's scores, gather)
    w64 = fold64(cache)
    for (l, h, b) in [(0, 0, 0), (0, 7, 0)]:
        parity.check_unit(cache, fused, l, h, b, w64, literal_subset=512)


def test_single_kernel_step_ragged_edges():
    lens = [0, 1, 127, 2048, 2049, 3000, 5000, 8192]
    wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=1, num_kv_heads=1, batch=len(lens))
    cache = gen.make_cache(wl, seed=52, device=DEV, lens=lens)
    fused, split = both_paths(cache, wl.budget)
    assert_same(cache, fused, split, wl.budget)
    w64 = fold64(cache)
    for b in range(len(lens)):
        parity.check_unit(cache, fused, 0, 0, b, w64, literal_subset=512)


def test_single_kernel_step_ties_across_slices():
    """Two distinct keys, one at 1000 random places and the other everywhere
    else: with B = 3000 one of the two fills the budget only in part, so the
    kept set ends in a run of equal scores whose lowest indices win, and that
    run spreads over several CTAs' slices (500 keys each).  NaN and +/-inf
    keys take part too."""
    wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=2, seq_len=8000)
    cache = gen.make_cache(wl, seed=53, device=DEV)
    rng = np.random.default_rng(53)
    qc = cache.query_center.reshape(-1, 128)
    for h in range(2):
        hi = qc[h].sign().to(torch.bfloat16)
        lo = (-qc[h].sign()).to(torch.bfloat16)
        rows = cache.k[0, h, 0]
        rows[:] = lo.to(DEV)
        pick = torch.from_numpy(rng.choice(8000, size=1000, replace=False)).to(DEV)
        rows[pick] = hi.to(DEV)
        rows[17] = float("nan")
        rows[18] = float("inf")
        rows[7000] = -float("inf")
    B = 3000
    fused, split = both_paths(cache, B)
    assert_same(cache, fused, split, B)
    for h in range(2):
        s = fused.scores[h, :8000].cpu().numpy()
        np.testing.assert_array_equal(fused.kept[h].cpu().numpy(), oracle.select(s, B))


@pytest.mark.parametrize("n,B", [(5000, 4999), (5000, 5000), (5000, 5001), (4096, 1), (300, 2048), (8192, 3000)])
def test_single_kernel_step_budget_edges(n, B):
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_kv_heads=3, seq_len=n)
    cache = gen.make_cache(wl, seed=54, device=DEV)
    fused, split = both_paths(cache, B)
    assert_same(cache, fused, split, B)


def test_single_kernel_step_is_taken_for_short_rows_only():
    import rope_aware_key_b200 as tri
    short = gen.make_cache(gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=2, seq_len=8192), seed=55,
                           device=DEV, with_values=True)
    n0 = tri.kernel_launches()
    parity.run_gpu(short, fused=True)
    assert tri.kernel_launches() - n0 == 2           # fold + one cluster kernel
    long = gen.make_cache(gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=2, seq_len=8193), seed=55,
                          device=DEV, with_values=True)
    n0 = tri.kernel_launches()
    parity.run_gpu(long, fused=True)
    assert tri.kernel_launches() - n0 == 4           # fold + score, select, compact
