"""The per-key-distance scorer (pre-RoPE caches) against the oracle's literal
offset average at each key's own distance, on the same seeded caches and
positions."""
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


def band_scale(keys_bits, w64, pairing):
    """sum_f |a_f| |k_f| per key: bounds |s| at any distance."""
    k = keys_bits.astype(np.uint32) << 16
    k = k.view(np.float32).astype(np.float64)
    if pairing == 0:
        kr, ki, ar, ai = k[:, :64], k[:, 64:], w64[:64], w64[64:]
    else:
        kr, ki, ar, ai = k[:, 0::2], k[:, 1::2], w64[0::2], w64[1::2]
    return np.hypot(kr, ki) @ np.hypot(ar, ai)


def run_pos(cache, positions, qpos, pairing=0):
    import rope_aware_key_b200 as tri
    wl = cache.wl
    qc = cache.query_center.reshape(-1, wl.head_dim).to(DEV).contiguous()
    w = tri.fold_weights(qc, wl.theta, wl.offsets, 0.0, pairing)
    d = parity.make_desc(cache)
    scores = torch.full((d.units, tri.score_row_stride(d)), float("nan"), device=DEV)
    tri.score_keys_at_positions(d, w, wl.theta, qpos, positions, pairing, scores)
    status = tri.read_device_status()
    torch.cuda.synchronize()
    return w, scores, status


def check_unit_pos(cache, scores, w64, positions, qpos, l, h, b, pairing, subset=None):
    wl = cache.wl
    u = parity.unit_id(wl, l, h, b)
    n = cache.lens[b]
    keys = parity.bits16(gen.unit_rows(cache, cache.k, l, h, b))
    s = scores[u, :n].cpu().numpy().astype(np.float64)
    p = np.arange(n, dtype=np.int64) if positions is None else positions[u, :n].cpu().numpy().astype(np.int64)
    if subset:
        idx = np.linspace(0, n - 1, num=min(n, subset)).astype(np.int64)
        keys, s, p = keys[idx], s[idx], p[idx]
    ref = oracle.score_at_positions(keys, cache.query_center[l, h].numpy(), wl.theta, wl.offsets, p, qpos[b],
                                    pairing)
    lh = l * wl.num_kv_heads + h
    scale = band_scale(keys, w64[lh], pairing)
    bad = np.flatnonzero(~(np.abs(s - ref) <= parity.SCORE_TOL * scale))
    assert bad.size == 0, (u, bad[:5], s[bad[:5]], ref[bad[:5]])
    return (float(np.max(np.abs(s - ref) / np.maximum(scale, 1e-300))) if n else 0.0), ref


def folded64(cache, pairing):
    wl = cache.wl
    return oracle.fold_w(cache.query_center.reshape(-1, wl.head_dim), wl.theta, wl.offsets, 0.0, pairing)


@pytest.mark.parametrize("pairing", [0, 1])
def test_positions_identity_contig(pairing):
    """No positions array: key i sits at position i; the query right after the last key."""
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=3, batch=2, seq_len=1000, theta=1e6)
    cache = gen.make_cache(wl, seed=31, device=DEV, with_values=False)
    qpos = [1000, 5000]
    w, scores, status = run_pos(cache, None, qpos, pairing)
    assert status == 0
    w64 = folded64(cache, pairing)
    worst = 0.0
    for l in range(2):
        for h in range(3):
            for b in range(2):
                worst = max(worst, check_unit_pos(cache, scores, w64, None, qpos, l, h, b, pairing)[0])
    assert worst < 1e-5
    assert torch.isnan(scores[:, 1000:]).all()          # row padding untouched


@pytest.mark.parametrize("pairing", [0, 1])
def test_positions_compacted_ragged_edges(pairing):
    wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=7)
    cache = gen.make_cache(wl, seed=32, device=DEV, with_values=False, lens=[1, 127, 128, 129, 300, 0, 2049])
    import rope_aware_key_b200 as tri
    stride = tri.score_row_stride(parity.make_desc(cache))
    positions, qpos = gen.key_positions(cache, seed=32, stride=stride)
    w, scores, status = run_pos(cache, positions, qpos, pairing)
    assert status == 0
    w64 = folded64(cache, pairing)
    for l in range(2):
        for h in range(2):
            for b in range(7):
                check_unit_pos(cache, scores, w64, positions, qpos, l, h, b, pairing)


def test_positions_paged():
    wl = gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=2, batch=5, len_lo=1, len_hi=700)
    cache = gen.make_cache(wl, seed=33, device=DEV, with_values=False)
    import rope_aware_key_b200 as tri
    stride = tri.score_row_stride(parity.make_desc(cache))
    positions, qpos = gen.key_positions(cache, seed=33, stride=stride, spread=3)
    w, scores, status = run_pos(cache, positions, qpos)
    assert status == 0
    w64 = folded64(cache, 0)
    for l in range(2):
        for h in range(wl.num_kv_heads):
            for b in range(5):
                check_unit_pos(cache, scores, w64, positions, qpos, l, h, b, 0)


def test_positions_far_negative_and_out_of_range():
    """Distances up to 2^31 - 1 either way are exact; beyond that the score is NaN and flagged."""
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["tiny"], seq_len=300, theta=5e5)
    cache = gen.make_cache(wl, seed=34, device=DEV, with_values=False)
    keys = parity.bits16(gen.unit_rows(cache, cache.k, 0, 0, 0))
    w64 = folded64(cache, 0)
    stride = tri.score_row_stride(parity.make_desc(cache))
    rng = np.random.default_rng(34)

    def run_with(p, t):
        positions = torch.full((1, stride), -1, dtype=torch.int32)
        positions[0, :300] = torch.from_numpy(p.astype(np.int32))
        w, scores, status = run_pos(cache, positions.to(DEV), [t])
        return scores[0, :300].cpu().numpy().astype(np.float64), status

    def check(s, p, t, good):
        ref = oracle.score_at_positions(keys[good], cache.query_center[0, 0].numpy(), wl.theta, wl.offsets,
                                        p[good], t)
        scale = band_scale(keys[good], w64[0], 0)
        assert np.all(np.abs(s[good] - ref) <= parity.SCORE_TOL * scale)

    # far behind the query: 0 < t - p <= 2^31 - 1; then 40 keys with t - p >= 2^31
    t = 2 ** 31 - 1
    p = rng.integers(0, 2 ** 31 - 1, size=300)
    p[260:299] = rng.integers(-2 ** 31 + 1, 0, size=39)
    p[299] = -1
    s, status = run_with(p, t)
    bad = np.arange(300) >= 260
    assert status == tri.DEVFLAG_BAD_POSITION
    assert np.isnan(s[bad]).all() and not np.isnan(s[~bad]).any()
    check(s, p, t, np.flatnonzero(~bad))
    # far ahead of the query: -2^31 < t - p < 0
    t = 1000
    p = rng.integers(1001, 2 ** 31 - 1, size=300)
    s, status = run_with(p, t)
    assert status == 0
    check(s, p, t, np.arange(300))
    # no positions array, query at 0: distances 0, -1, -2, ...
    w, scores, status = run_pos(cache, None, [0])
    assert status == 0
    check_unit_pos(cache, scores, w64, None, [0], 0, 0, 0, 0)


def test_positions_select_and_compact():
    """Selection on the distance scores: exact against the oracle's selection on
    the GPU's own fp32 scores, and within the tie band of the fp64 reference;
    the compacted rows are the kept rows."""
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_kv_heads=2)
    cache = gen.make_cache(wl, seed=35, device=DEV)
    stride = tri.score_row_stride(parity.make_desc(cache))
    positions, qpos = gen.key_positions(cache, seed=35, stride=stride, spread=8)
    w, scores, status = run_pos(cache, positions, qpos)
    assert status == 0
    d = parity.make_desc(cache)
    B = wl.budget
    kept, cnt = tri.select_topk(d, scores, B)
    k_out = torch.zeros((d.units, B, 128), dtype=torch.bfloat16, device=DEV)
    v_out = torch.zeros_like(k_out)
    tri.compact_kv(d, kept, cnt, B, tri.COMPACT_OUT_OF_PLACE, k_out, v_out)
    torch.cuda.synchronize()
    w64 = folded64(cache, 0)
    for h in range(2):
        u = parity.unit_id(wl, 0, h, 0)
        _, ref = check_unit_pos(cache, scores, w64, positions, qpos, 0, h, 0, 0)
        keys = parity.bits16(gen.unit_rows(cache, cache.k, 0, h, 0))
        scale = band_scale(keys, w64[h], 0)
        s = scores[u, :wl.seq_len].cpu().numpy()
        kp = kept[u].cpu().numpy()
        np.testing.assert_array_equal(kp, oracle.select(s, B))
        top = oracle.select(ref, B)
        sB = ref[top].min()
        eps = parity.SCORE_TOL * scale
        amb = np.abs(ref - sB) <= eps + eps[top[np.argmin(ref[top])]]
        inside = np.zeros(wl.seq_len, bool)
        inside[kp] = True
        assert np.all(inside[(ref > sB) & ~amb]) and not np.any(inside[(ref < sB) & ~amb])
        rows = gen.unit_rows(cache, cache.k, 0, h, 0)
        assert torch.equal(k_out[u], rows[kept[u].long()])
        assert torch.equal(v_out[u], gen.unit_rows(cache, cache.v, 0, h, 0)[kept[u].long()])


def test_positions_full_qwen3_sampled():
    """The 36 x 8 x 32768 cache scored at positions 0..32767 with the query at 32768."""
    wl = gen.WORKLOADS["qwen3_full"]
    cache = gen.make_cache(wl, seed=0, device=DEV, with_values=False)
    qpos = [wl.seq_len]
    w, scores, status = run_pos(cache, None, qpos)
    assert status == 0
    w64 = folded64(cache, 0)
    for (l, h) in [(0, 0), (17, 5), (35, 7)]:
        check_unit_pos(cache, scores, w64, None, qpos, l, h, 0, 0, subset=2048)
    assert not torch.isnan(scores).any()


@pytest.mark.parametrize("pairing", [0, 1])
def test_positions_unpacked_contig(pairing):
    """A cache whose sequences are padded (not packed back to back) takes the
    general scorer; it must agree with the oracle like the packed one."""
    import rope_aware_key_b200 as tri
    wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=2, batch=2, seq_len=700, theta=1e6)
    cache = gen.make_cache(wl, seed=36, device=DEV, with_values=False)
    padded = torch.zeros((2, 2, 2, 712, 128), dtype=torch.bfloat16, device=DEV)
    padded[..., :700, :] = cache.k
    view = padded[..., :700, :]
    d = tri.desc_contig(view, None)
    qc = cache.query_center.reshape(-1, 128).to(DEV).contiguous()
    w = tri.fold_weights(qc, wl.theta, wl.offsets, 0.0, pairing)
    stride = tri.score_row_stride(d)
    positions, qpos = gen.key_positions(cache, seed=36, stride=stride, spread=5)
    scores = torch.full((d.units, stride), float("nan"), device=DEV)
    tri.score_keys_at_positions(d, w, wl.theta, qpos, positions, pairing, scores)
    assert tri.read_device_status() == 0
    # the same cache packed: the fast scorer
    packed = torch.full_like(scores, float("nan"))
    tri.score_keys_at_positions(tri.desc_contig(cache.k, None), w, wl.theta, qpos, positions, pairing, packed)
    torch.cuda.synchronize()
    w64 = folded64(cache, pairing)
    for l in range(2):
        for h in range(2):
            for b in range(2):
                check_unit_pos(cache, scores, w64, positions, qpos, l, h, b, pairing)
                check_unit_pos(cache, packed, w64, positions, qpos, l, h, b, pairing)
