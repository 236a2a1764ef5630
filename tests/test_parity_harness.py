"""The parity checker itself, on the CPU: results built from the oracle pass,
and results with a planted mistake fail.  (The GPU tests rely on it.)"""
import numpy as np
import pytest
import torch

import gen
import oracle
from tests import parity


def fake_result(cache, B, mode=0, perturb=None):
    """A GpuResult computed by the oracle (fp32 scores), as the GPU would give."""
    wl = cache.wl
    w64 = oracle.fold_w(cache.query_center.reshape(-1, wl.head_dim), wl.theta, wl.offsets)
    units = wl.units
    stride = (max(cache.lens) + 3) // 4 * 4
    scores = torch.full((units, stride), float("nan"))
    kept = torch.full((units, B), -7, dtype=torch.int32)
    cnt = torch.zeros(units, dtype=torch.int32)
    k_out = torch.zeros((units, B, wl.head_dim), dtype=torch.bfloat16)
    v_out = torch.zeros_like(k_out)
    for l in range(wl.num_layers):
        for h in range(wl.num_kv_heads):
            for b in range(wl.batch):
                u = parity.unit_id(wl, l, h, b)
                keys = parity.bits16(gen.unit_rows(cache, cache.k, l, h, b))
                vals = parity.bits16(gen.unit_rows(cache, cache.v, l, h, b))
                s = oracle.score_realdot(keys, w64[l * wl.num_kv_heads + h]).astype(np.float32)
                if perturb == "score" and u == 0:
                    s[3] += np.float32(abs(s[3]) * 1e-2 + 1.0)
                n = len(s)
                scores[u, :n] = torch.from_numpy(s)
                kk = oracle.select(s, B)
                if perturb == "kept" and u == 0:
                    kk = kk.copy()
                    kk[-1] = np.setdiff1d(np.arange(n), kk)[0] if n > B else kk[-1]
                    kk.sort()
                kept[u, :len(kk)] = torch.from_numpy(kk)
                cnt[u] = len(kk)
                ko = oracle.gather_rows(keys, kk)
                if perturb == "row" and u == 0:
                    ko = ko.copy()
                    ko[0, 5] ^= 1
                k_out[u, :len(kk)] = torch.from_numpy(ko.view(np.int16)).view(torch.bfloat16)
                v_out[u, :len(kk)] = torch.from_numpy(oracle.gather_rows(vals, kk).view(np.int16)).view(torch.bfloat16)
    w = torch.from_numpy(w64.astype(np.float32))
    return parity.GpuResult(w, scores, kept, cnt, k_out, v_out, 0, B, mode), w64


def small_cache(layout="contig"):
    if layout == "contig":
        wl = gen.scaled(gen.WORKLOADS["tiny"], num_layers=2, num_kv_heads=2, batch=2, seq_len=300, budget=64)
    else:
        wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=1, num_kv_heads=2, batch=3, len_lo=20,
                        len_hi=200, budget=64)
    return gen.make_cache(wl, seed=0, device="cpu")


@pytest.mark.parametrize("layout", ["contig", "ragged"])
def test_checker_accepts_oracle_results(layout):
    c = small_cache(layout)
    res, w64 = fake_result(c, 64)
    parity.check_fold(res, c)
    for l in range(c.wl.num_layers):
        for h in range(c.wl.num_kv_heads):
            for b in range(c.wl.batch):
                rep = parity.check_unit(c, res, l, h, b, w64[l * c.wl.num_kv_heads + h], literal=True)
                assert rep.max_err_over_l1 < 1e-6
    parity.check_all_units_properties(c, res)


@pytest.mark.parametrize("perturb", ["score", "kept", "row"])
def test_checker_rejects_planted_mistakes(perturb):
    c = small_cache()
    res, w64 = fake_result(c, 64, perturb=perturb)
    with pytest.raises(AssertionError):
        parity.check_unit(c, res, 0, 0, 0, w64[0], literal=False)


def test_checker_holefill_mode():
    c = gen.make_cache(gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=1, num_kv_heads=4, batch=3,
                                  len_lo=10, len_hi=90, budget=32, spare_blocks_per_seq=0), seed=1, device="cpu")
    res, w64 = fake_result(c, 32, mode=1)
    res.k_out = res.v_out = None
    for h in range(4):
        for b in range(3):
            keys = parity.bits16(gen.unit_rows(c, c.k, 0, h, b))
            vals = parity.bits16(gen.unit_rows(c, c.v, 0, h, b))
            kk = res.kept[parity.unit_id(c.wl, 0, h, b), :res.kept_count[parity.unit_id(c.wl, 0, h, b)]].numpy()
            ak, _ = oracle.holefill(keys, kk, 32)
            av, _ = oracle.holefill(vals, kk, 32)
            parity.check_unit(c, res, 0, h, b, w64[h], before_k=keys, before_v=vals, after_k=ak, after_v=av)
            bad = ak.copy()
            if len(bad) > 32:
                bad[0, 0] ^= 1
                with pytest.raises(AssertionError):
                    parity.check_unit(c, res, 0, h, b, w64[h], before_k=keys, before_v=vals, after_k=bad,
                                      after_v=av)


def test_generator_recipe():
    """The generator's draws follow the stated recipe (seeded, shapes, outliers)."""
    wl = gen.scaled(gen.WORKLOADS["qwen3_layer"], num_kv_heads=2, seq_len=20000)
    c1 = gen.make_cache(wl, seed=0, device="cpu")
    c2 = gen.make_cache(wl, seed=0, device="cpu")
    assert torch.equal(c1.k.view(torch.int16), c2.k.view(torch.int16))
    k = c1.k[0, 0, 0].float()
    norm = k.norm(dim=1)
    base = c1.key_center[0, 0].norm()
    outl = (norm > 2.5 * base)
    assert 0.005 < outl.float().mean().item() < 0.02          # ~1% outliers x5
    ratio = (norm[outl] / base).mean().item()
    assert 4.5 < ratio < 5.5
    spread = (k[~outl] - c1.key_center[0, 0]).std().item()
    assert abs(spread - wl.sigma) < 0.02
    lens = gen.seq_lengths(gen.WORKLOADS["qwen3_ragged"], 0)
    assert len(lens) == 8 and all(8192 <= n <= 32768 for n in lens)


def test_key_positions_recipe():
    """Positions of a compacted pre-RoPE cache: per unit sorted, distinct, inside
    [0, spread * n), padded with -1, seeded."""
    wl = gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=2, num_kv_heads=2, batch=3)
    c = gen.make_cache(wl, seed=5, device="cpu", with_values=False, lens=[5, 0, 300])
    pos, qpos = gen.key_positions(c, seed=5, stride=304, spread=3)
    assert pos.shape == (12, 304) and qpos == [15, 0, 900]
    for u in range(12):
        b = u % 3
        n = c.lens[b]
        row = pos[u].numpy()
        assert (row[n:] == -1).all()
        assert (np.diff(row[:n]) > 0).all() and (row[:n] >= 0).all() and (row[:n] < qpos[b]).all()
    again, _ = gen.key_positions(c, seed=5, stride=304, spread=3)
    assert torch.equal(pos, again)
    assert not torch.equal(pos[2], pos[5])           # units draw independently


@pytest.mark.parametrize("layout", ["contig", "ragged", "paged"])
def test_generator_layer_range_is_a_slice_of_the_whole(layout):
    """A rank that holds layers l0..l1-1 of a cache draws exactly those layers
    of the whole cache (keys, values, centers, appended tokens)."""
    base = {"contig": gen.scaled(gen.WORKLOADS["tiny"], num_layers=5, num_kv_heads=2, batch=2, seq_len=40),
            "ragged": gen.scaled(gen.WORKLOADS["qwen3_ragged"], num_layers=5, num_kv_heads=2, batch=3),
            "paged": gen.scaled(gen.WORKLOADS["qwen25_paged"], num_layers=5, num_kv_heads=2, batch=3,
                                spare_blocks_per_seq=2)}[layout]
    lens = None if layout == "contig" else [30, 17, 64]
    whole = gen.make_cache(base, seed=3, device="cpu", lens=lens)
    part = gen.make_cache(base, seed=3, device="cpu", lens=lens, layer_range=(2, 4))
    assert part.wl.num_layers == 2 and part.layer0 == 2
    assert torch.equal(part.key_center, whole.key_center[2:4])
    assert torch.equal(part.query_center, whole.query_center[2:4])
    for l in range(2):
        for h in range(base.num_kv_heads):
            for b in range(base.batch):
                for t in ("k", "v"):
                    a = gen.unit_rows(part, getattr(part, t), l, h, b)
                    w = gen.unit_rows(whole, getattr(whole, t), 2 + l, h, b)
                    assert torch.equal(a.view(torch.int16), w.view(torch.int16))
    if layout == "paged":
        gen.append_tokens(whole, 16, step=1)
        gen.append_tokens(part, 16, step=1)
        for b in range(base.batch):
            a = gen.unit_rows(part, part.k, 1, 0, b)[-16:]
            w = gen.unit_rows(whole, whole.k, 3, 0, b)[-16:]
            assert torch.equal(a.view(torch.int16), w.view(torch.int16))
