"""Parity harness: run the CUDA path through the C ABI and compare it, unit by
unit, with the CPU oracle on the same seeded inputs.

Bars:
* scores: |s_gpu - s_ref| <= 1e-4 * sum_j |w_j k_j| per key, s_ref the
  oracle's literal per-offset average (or its folded form, pinned equal to
  it on the CPU, where the literal one is too slow);
* selection: bit-exact against the oracle's selection run on the GPU's own
  fp32 scores (both sides decide in fp32), and, against the fp64 reference,
  exact except for keys whose reference score lies within the score
  tolerance of the B-th score;
* compaction: bit-exact against a gather (or hole fill) at the GPU's own
  kept indices.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

import gen
import oracle

SCORE_TOL = 1e-4


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (numpy, on the host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def unit_id(wl: gen.Workload, l: int, h: int, b: int) -> int:
    return (l * wl.num_kv_heads + h) * wl.batch + b


def make_desc(cache: gen.Cache, max_seq_len: int = 0):
    import rope_aware_key_b200 as tri
    wl = cache.wl
    if wl.layout == "contig":
        return tri.desc_contig(cache.k, cache.v, max_seq_len=max_seq_len)
    if wl.layout == "ragged":
        return tri.desc_ragged(cache.k, cache.v, cache.cu_seqlens.cpu().tolist(), max_seq_len=max_seq_len)
    return tri.desc_paged(cache.k, cache.v, cache.block_table, cache.lens, max_seq_len=max_seq_len)


@dataclasses.dataclass
class GpuResult:
    w: torch.Tensor
    scores: torch.Tensor
    kept: torch.Tensor
    kept_count: torch.Tensor
    k_out: Optional[torch.Tensor]
    v_out: Optional[torch.Tensor]
    status: int
    budget: int
    mode: int


def run_gpu(cache: gen.Cache, budget: Optional[int] = None, pairing: int = 0, delta0: Optional[float] = None,
            mode: int = 0, fused: bool = False, max_seq_len: int = 0) -> GpuResult:
    """fold -> score -> select -> compact through the C ABI (all on the device)."""
    import rope_aware_key_b200 as tri
    wl = cache.wl
    B = budget or wl.budget
    dev = cache.k.device
    d0 = wl.delta0 if delta0 is None else delta0
    qc = cache.query_center.reshape(-1, wl.head_dim).to(dev).contiguous()
    w = tri.fold_weights(qc, wl.theta, wl.offsets, d0, pairing)
    d = make_desc(cache, max_seq_len)
    k_out = v_out = None
    if mode == tri.COMPACT_OUT_OF_PLACE:
        k_out = torch.zeros((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=dev)
        v_out = torch.zeros_like(k_out)
    scores = torch.full((d.units, tri.score_row_stride(d)), float("nan"), dtype=torch.float32, device=dev)
    kept = torch.full((d.units, B), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((d.units,), -7, dtype=torch.int32, device=dev)
    if fused:
        ws = torch.empty(tri.workspace_size(d, B), dtype=torch.uint8, device=dev)
        tri.compress(d, w, B, mode, kept, cnt, k_out, v_out, ws)
        stride = tri.score_row_stride(d)
        scores.copy_(ws[: d.units * stride * 4].view(torch.float32).view(d.units, stride))
    else:
        tri.score_keys(d, w, scores)
        tri.select_topk(d, scores, B, kept, cnt)
        tri.compact_kv(d, kept, cnt, B, mode, k_out, v_out)
    status = tri.read_device_status(clear=True)
    torch.cuda.synchronize()
    return GpuResult(w, scores, kept, cnt, k_out, v_out, status, B, mode)


@dataclasses.dataclass
class UnitReport:
    unit: int
    n: int
    max_err_over_l1: float
    ambiguous: int


def check_scores(keys_bits: np.ndarray, s_gpu: np.ndarray, ref: np.ndarray, w64: np.ndarray):
    """Per-key bar |s_gpu - ref| <= 1e-4 * sum_j |w_j k_j|; returns (max ratio, L1)."""
    l1 = oracle.abs_dot(keys_bits, w64)
    err = np.abs(s_gpu.astype(np.float64) - ref)
    ratio = err / np.maximum(l1, 1e-300)
    bad = np.flatnonzero(err > SCORE_TOL * l1)
    assert bad.size == 0, f"{bad.size} scores off, first {bad[:5]}: gpu {s_gpu[bad[:5]]} ref {ref[bad[:5]]}"
    return float(ratio.max()) if ratio.size else 0.0, l1


def check_selection(s_gpu: np.ndarray, kept: np.ndarray, ref: np.ndarray, l1: np.ndarray, B: int) -> int:
    """Returns the number of ambiguous keys (within tolerance of the B-th score)."""
    n = s_gpu.shape[0]
    m = min(B, n)
    assert kept.shape[0] == m
    # exact: same decision in fp32
    want = oracle.select(s_gpu.astype(np.float32), B)
    np.testing.assert_array_equal(kept, want)
    if n <= B:
        return 0
    # against the fp64 reference, up to the tie band
    top = oracle.select(ref, B)
    sB = ref[top].min()
    iB = top[np.argmin(ref[top])]
    eps = SCORE_TOL * l1
    amb = np.abs(ref - sB) <= eps + eps[iB]
    keptset = np.zeros(n, dtype=bool)
    keptset[kept] = True
    must_in = (ref > sB) & ~amb
    must_out = (ref < sB) & ~amb
    assert np.all(keptset[must_in]), np.flatnonzero(must_in & ~keptset)[:10]
    assert not np.any(keptset[must_out]), np.flatnonzero(must_out & keptset)[:10]
    return int(amb.sum())


def check_unit(cache: gen.Cache, res: GpuResult, l: int, h: int, b: int, w64: np.ndarray,
               literal: bool = True, literal_subset: Optional[int] = None, pairing: int = 0,
               delta0: Optional[float] = None, before_k: Optional[np.ndarray] = None,
               before_v: Optional[np.ndarray] = None, after_k: Optional[np.ndarray] = None,
               after_v: Optional[np.ndarray] = None) -> UnitReport:
    """All checks for one unit.  For the in-place mode pass the unit's rows
    before and after compaction (host uint16 arrays)."""
    wl = cache.wl
    u = unit_id(wl, l, h, b)
    n = cache.lens[b]
    B = res.budget
    d0 = wl.delta0 if delta0 is None else delta0
    keys = before_k if before_k is not None else bits16(gen.unit_rows(cache, cache.k, l, h, b))
    s_gpu = res.scores[u, :n].cpu().numpy()
    qc = cache.query_center[l, h].numpy()
    if literal:
        ref = oracle.score_literal(keys, qc, wl.theta, wl.offsets, d0, pairing)
    else:
        ref = oracle.score_folded(keys, qc, wl.theta, wl.offsets, d0, pairing)
        if literal_subset:
            idx = np.linspace(0, n - 1, num=min(n, literal_subset)).astype(np.int64)
            lit = oracle.score_literal(keys[idx], qc, wl.theta, wl.offsets, d0, pairing)
            check_scores(keys[idx], s_gpu[idx], lit, w64)
    ratio, l1 = check_scores(keys, s_gpu, ref, w64)

    cnt = int(res.kept_count[u])
    assert cnt == min(B, n), (cnt, B, n)
    kept = res.kept[u, :cnt].cpu().numpy()
    amb = check_selection(s_gpu, kept, ref, l1, B)

    import rope_aware_key_b200 as tri
    if res.mode == tri.COMPACT_OUT_OF_PLACE:
        vals = before_v if before_v is not None else bits16(gen.unit_rows(cache, cache.v, l, h, b))
        np.testing.assert_array_equal(bits16(res.k_out[u, :cnt]), oracle.gather_rows(keys, kept))
        np.testing.assert_array_equal(bits16(res.v_out[u, :cnt]), oracle.gather_rows(vals, kept))
    else:
        assert before_v is not None and after_k is not None and after_v is not None
        exp_k, moved = oracle.holefill(keys, kept, B)
        exp_v, _ = oracle.holefill(before_v, kept, B)
        np.testing.assert_array_equal(after_k, exp_k)
        np.testing.assert_array_equal(after_v, exp_v)
    return UnitReport(u, n, ratio, amb)


def check_fold(res: GpuResult, cache: gen.Cache, pairing: int = 0, delta0: Optional[float] = None) -> np.ndarray:
    """The device fold against the oracle's fp64 2x2 map; returns the fp64 weights."""
    wl = cache.wl
    d0 = wl.delta0 if delta0 is None else delta0
    w64 = oracle.fold_w(cache.query_center.reshape(-1, wl.head_dim), wl.theta, wl.offsets, d0, pairing)
    wg = res.w.cpu().numpy().astype(np.float64)
    err = np.abs(wg - w64)
    tol = 2.0 ** -23 * np.abs(w64) + 1e-12 * np.abs(w64).max()
    assert np.all(err <= tol), float((err / np.maximum(np.abs(w64), 1e-30)).max())
    return w64


def check_all_units_properties(cache: gen.Cache, res: GpuResult) -> None:
    """Properties that hold at any size, checked on every unit on the device
    with plain torch ops: counts, ascending in-range indices, and every kept
    score >= every evicted score (no NaNs in the synthetic inputs)."""
    wl = cache.wl
    B = res.budget
    lens = torch.tensor(cache.lens, device=res.kept.device, dtype=torch.int32)
    n_u = lens.repeat(wl.num_layers * wl.num_kv_heads)            # unit u -> its sequence's length
    assert torch.equal(res.kept_count, torch.minimum(n_u, torch.tensor(B, device=n_u.device, dtype=torch.int32)))
    stride = res.scores.shape[1]
    col = torch.arange(B, device=res.kept.device)
    valid = col[None, :] < res.kept_count[:, None]
    k = res.kept.long()
    assert torch.all((k >= 0)[valid]) and torch.all((k < n_u[:, None])[valid])
    diffs = k[:, 1:] - k[:, :-1]
    assert torch.all((diffs > 0)[valid[:, 1:]])
    scores = res.scores
    keys_valid = torch.arange(stride, device=scores.device)[None, :] < n_u[:, None]
    hits = torch.zeros(keys_valid.shape, dtype=torch.int32, device=scores.device)
    hits.scatter_add_(1, torch.where(valid, k, 0), valid.to(torch.int32))
    is_kept = hits > 0
    neg = torch.tensor(float("-inf"), device=scores.device)
    pos = torch.tensor(float("inf"), device=scores.device)
    min_kept = torch.where(is_kept, scores, pos).min(dim=1).values
    max_ev = torch.where(keys_valid & ~is_kept, scores, neg).max(dim=1).values
    assert torch.all(min_kept >= max_ev)
    if res.k_out is not None and wl.layout == "contig":
        # out-of-place rows equal a plain torch gather, on every unit
        N = cache.lens[0]
        for src, out in ((cache.k, res.k_out), (cache.v, res.v_out)):
            flat = src.view(-1, N, wl.head_dim)
            idx = torch.where(valid, k, 0)[:, :, None].expand(-1, -1, wl.head_dim)
            want = torch.gather(flat, 1, idx).view(torch.int16)
            got = out.view(torch.int16)
            assert torch.equal(torch.where(valid[:, :, None], got, 0), torch.where(valid[:, :, None], want, 0))
