"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host (before any CUDA
call) with the documented status codes."""
import ctypes
import os
import re

import pytest

import rope_aware_key_b200 as tri
from rope_aware_key_b200 import build as tri_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tri_evict.h")

FAKE = 0x10000          # an aligned non-null address; never dereferenced on the host


@pytest.fixture(scope="module")
def L():
    tri_build.build()
    return tri.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tri_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "tri_score_keys" in names and len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_exported_dynamic_symbols_match_header():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", tri.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(set(re.findall(r"\bT (tri_[a-z_0-9]+)\b", out)))
    assert exported == declared_functions()


def test_status_strings_and_version(L):
    for code, name in tri._STATUS.items():
        assert L.tri_status_string(code).decode() == name
    assert L.tri_version().decode().count(".") == 2


def contig(**kw):
    base = dict(layout=0, num_layers=2, num_kv_heads=8, head_dim=128, batch=1, max_seq_len=0, k=FAKE, v=FAKE,
                stride_layer=8 * 1000 * 128, stride_head=1000 * 128, stride_seq=1000 * 128, seq_len=1000)
    base.update(kw)
    return tri._CacheDesc(**base)


def test_row_stride_and_workspace(L):
    d = contig()
    assert L.tri_score_row_stride(ctypes.byref(d)) == 1000
    d = contig(seq_len=1001)
    assert L.tri_score_row_stride(ctypes.byref(d)) == 1004
    d = contig(seq_len=1001, max_seq_len=2000)
    assert L.tri_score_row_stride(ctypes.byref(d)) == 2000
    n = ctypes.c_size_t(0)
    assert L.tri_workspace_size(ctypes.byref(contig()), 64, ctypes.byref(n)) == 0
    assert n.value == 2 * 8 * 1000 * 4 + 256


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), 2),
    (dict(k=None), 1),
    (dict(k=FAKE + 8), 1),
    (dict(num_layers=0), 1),
    (dict(batch=300, stride_seq=128), 2),
    (dict(seq_len=-1), 1),
    (dict(stride_head=100), 1),
    (dict(stride_layer=0), 1),
    (dict(max_seq_len=10), 1),
    (dict(layout=7), 1),
])
def test_descriptor_rejected(L, kw, code):
    d = contig(**kw)
    assert L.tri_score_keys(ctypes.byref(d), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None) == code


def test_ragged_checks(L):
    cu = (ctypes.c_int32 * 4)(0, 10, 5, 20)       # not monotone
    d = tri._CacheDesc(layout=1, num_layers=1, num_kv_heads=1, head_dim=128, batch=3, k=FAKE, v=FAKE,
                       stride_layer=20 * 128, stride_head=20 * 128,
                       cu_seqlens=ctypes.cast(cu, ctypes.POINTER(ctypes.c_int32)))
    assert L.tri_score_keys(ctypes.byref(d), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None) == 1
    cu2 = (ctypes.c_int32 * 4)(1, 10, 15, 20)      # must start at 0
    d.cu_seqlens = ctypes.cast(cu2, ctypes.POINTER(ctypes.c_int32))
    assert L.tri_score_keys(ctypes.byref(d), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None) == 1
    cu3 = (ctypes.c_int32 * 4)(0, 10, 15, 21)
    d.cu_seqlens = ctypes.cast(cu3, ctypes.POINTER(ctypes.c_int32))
    assert L.tri_score_row_stride(ctypes.byref(d)) == 12
    # offsets whose int32 difference wraps: the third length would come out as
    # 11, starting below the buffer; it must be refused
    cu4 = (ctypes.c_int32 * 4)(0, 1 << 30, (1 << 31) - 1, -(1 << 31) + 10)
    d.cu_seqlens = ctypes.cast(cu4, ctypes.POINTER(ctypes.c_int32))
    assert L.tri_score_row_stride(ctypes.byref(d)) == -1
    assert L.tri_score_keys(ctypes.byref(d), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None) == 1


def paged(**kw):
    lens = kw.pop("lens", (40, 17))
    arr = (ctypes.c_int32 * len(lens))(*lens)
    base = dict(layout=2, num_layers=1, num_kv_heads=4, head_dim=128, batch=len(lens), k=FAKE, v=FAKE,
                stride_layer=100 * 16 * 4 * 128, stride_block=16 * 4 * 128, block_table=FAKE,
                max_blocks_per_seq=4, block_size=16, num_blocks=100,
                seq_lens=ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)))
    base.update(kw)
    d = tri._CacheDesc(**base)
    d._arr = arr
    return d


@pytest.mark.parametrize("kw,code", [
    (dict(num_kv_heads=3, stride_block=16 * 3 * 128, stride_layer=100 * 16 * 3 * 128), 2),   # H must divide 8
    (dict(block_size=64), 2),                     # block_size * H > 128
    (dict(num_kv_heads=8, block_size=1 << 29, stride_block=1 << 39, stride_layer=1 << 40), 2),   # product wraps int32
    (dict(stride_block=16 * 4 * 128 - 8), 1),     # pages overlap
    (dict(lens=(65, 1)), 1),                      # longer than max_blocks * block_size
    (dict(block_table=None), 1),
    (dict(num_blocks=0), 1),
])
def test_paged_rejected(L, kw, code):
    d = paged(**kw)
    assert L.tri_score_keys(ctypes.byref(d), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None) == code


def test_select_and_compact_args(L):
    d = contig()
    P = ctypes.c_void_p
    assert L.tri_select_topk(ctypes.byref(d), P(FAKE), 0, P(FAKE), P(FAKE), None) == 1        # B < 1
    assert L.tri_select_topk(ctypes.byref(d), P(FAKE), 8, None, P(FAKE), None) == 1
    assert L.tri_compact_kv(ctypes.byref(d), P(FAKE), P(FAKE), 8, 0, None, P(FAKE), None) == 1   # no k_out
    assert L.tri_compact_kv(ctypes.byref(d), P(FAKE), P(FAKE), 8, 1, P(FAKE), None, None) == 1   # in place + out
    assert L.tri_compact_kv(ctypes.byref(d), P(FAKE), P(FAKE), 8, 5, P(FAKE), P(FAKE), None) == 1
    dv = contig(v=None)
    assert L.tri_compact_kv(ctypes.byref(dv), P(FAKE), P(FAKE), 8, 0, P(FAKE), P(FAKE), None) == 1


def test_compress_workspace_checked_on_host(L):
    d = contig()
    P = ctypes.c_void_p
    need = ctypes.c_size_t(0)
    L.tri_workspace_size(ctypes.byref(d), 64, ctypes.byref(need))
    st = L.tri_compress(ctypes.byref(d), P(FAKE), 64, 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                        need.value - 1, None)
    assert st == 3
    st = L.tri_compress(ctypes.byref(d), P(FAKE), 64, 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE + 16),
                        need.value, None)
    assert st == 1      # workspace not 256-byte aligned


def test_compress_max_checked_on_host(L):
    """tri_compress_max: its workspace, the max scorer's limits and the
    compaction's checks are made before anything is launched (no GPU here)."""
    d = contig()
    P = ctypes.c_void_p
    need = ctypes.c_size_t(0)
    L.tri_workspace_size(ctypes.byref(d), 64, ctypes.byref(need))
    n0 = L.tri_kernel_launches()
    args = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert L.tri_compress_max(ctypes.byref(d), P(FAKE), 17, 64, 0, *args, need.value - 1, None) == 3
    assert L.tri_compress_max(ctypes.byref(d), P(FAKE), 17, 64, 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                              P(FAKE + 16), need.value, None) == 1      # workspace not 256-byte aligned
    assert L.tri_compress_max(ctypes.byref(d), P(FAKE), 65, 64, 0, *args, need.value, None) == 2   # offsets
    assert L.tri_compress_max(ctypes.byref(d), P(FAKE), 0, 64, 0, *args, need.value, None) == 1
    assert L.tri_compress_max(ctypes.byref(d), P(FAKE), 17, 0, 0, *args, need.value, None) == 1    # B < 1
    loose = contig(stride_head=1000 * 128 + 64, stride_layer=8 * (1000 * 128 + 64))
    L.tri_workspace_size(ctypes.byref(loose), 64, ctypes.byref(need))
    assert L.tri_compress_max(ctypes.byref(loose), P(FAKE), 17, 64, 0, *args, need.value, None) == 2  # not packed
    pg = paged(block_size=12, stride_block=12 * 4 * 128, stride_layer=100 * 12 * 4 * 128)
    L.tri_workspace_size(ctypes.byref(pg), 8, ctypes.byref(need))
    assert L.tri_compress_max(ctypes.byref(pg), P(FAKE), 17, 8, 1, P(FAKE), P(FAKE), None, None, P(FAKE),
                              need.value, None) == 2                                        # pages of 12
    assert L.tri_kernel_launches() == n0


def test_compress_refuses_before_any_launch(L):
    """More score tiles than an int32 counts (65536 heads x 2^24 keys) is
    refused by both compress calls before the scorer runs: the status is
    TRI_ERR_UNSUPPORTED and no kernel was launched (no CUDA call is made
    either, which is why this runs without a GPU)."""
    n, H = 1 << 24, 1 << 16
    d = contig(num_layers=1, num_kv_heads=H, seq_len=n, stride_layer=H * n * 128, stride_head=n * 128,
               stride_seq=n * 128)
    P = ctypes.c_void_p
    need = ctypes.c_size_t(0)
    assert L.tri_workspace_size(ctypes.byref(d), 2048, ctypes.byref(need)) == 0
    n0 = L.tri_kernel_launches()
    assert L.tri_score_keys(ctypes.byref(d), P(FAKE), P(FAKE), None) == 2
    for mode, ko in ((0, FAKE), (1, None)):
        st = L.tri_compress(ctypes.byref(d), P(FAKE), 2048, mode, P(FAKE), P(FAKE), P(ko), P(ko), P(FAKE),
                            need.value, None)
        assert st == 2
    assert L.tri_kernel_launches() == n0


def test_compress_refuses_a_row_the_selection_cannot_hold(L):
    """A row too long for the selection's shared memory (2^20 keys at
    B = 2048) is refused by the selection and by both compress calls before
    the scorer runs: TRI_ERR_UNSUPPORTED, and no kernel launched."""
    n = 1 << 20
    d = contig(num_layers=1, num_kv_heads=1, seq_len=n, stride_layer=n * 128, stride_head=n * 128,
               stride_seq=n * 128)
    P = ctypes.c_void_p
    need = ctypes.c_size_t(0)
    assert L.tri_workspace_size(ctypes.byref(d), 2048, ctypes.byref(need)) == 0
    n0 = L.tri_kernel_launches()
    assert L.tri_select_topk(ctypes.byref(d), P(FAKE), 2048, P(FAKE), P(FAKE), None) == 2
    for mode, ko in ((0, FAKE), (1, None)):
        st = L.tri_compress(ctypes.byref(d), P(FAKE), 2048, mode, P(FAKE), P(FAKE), P(ko), P(ko), P(FAKE),
                            need.value, None)
        assert st == 2
        st = L.tri_compress_noalloc(ctypes.byref(d), P(FAKE), 2048, mode, P(FAKE), P(FAKE), P(ko), P(ko), None)
        assert st == 2
    assert L.tri_kernel_launches() == n0


def test_compress_refuses_oversized_gather_before_any_launch(L):
    """units x B past int32 (the gather's row count) is refused on the host."""
    d = contig(num_layers=1, num_kv_heads=8, batch=256, seq_len=4, stride_layer=8 * 256 * 4 * 128,
               stride_head=256 * 4 * 128, stride_seq=4 * 128)
    P = ctypes.c_void_p
    B = (1 << 31) // (8 * 256) + 1
    need = ctypes.c_size_t(0)
    assert L.tri_workspace_size(ctypes.byref(d), B, ctypes.byref(need)) == 0
    n0 = L.tri_kernel_launches()
    assert L.tri_compress(ctypes.byref(d), P(FAKE), B, 0, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                          need.value, None) == 2
    assert L.tri_kernel_launches() == n0


def fold_params(**kw):
    offs = kw.pop("offs", [1.0, 2.0, 4.0])
    arr = (ctypes.c_double * max(1, len(offs)))(*offs)
    base = dict(head_dim=128, theta=1e4, offsets=ctypes.cast(arr, ctypes.POINTER(ctypes.c_double)),
                n_offsets=len(offs), delta0=0.0, pairing=0)
    base.update(kw)
    p = tri._FoldParams(**base)
    p._arr = arr
    return p


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), 2),
    (dict(theta=0.0), 1),
    (dict(theta=float("nan")), 1),
    (dict(offs=[]), 1),
    (dict(offs=[1.0, float("inf")]), 1),
    (dict(n_offsets=5000), 2),
    (dict(pairing=3), 1),
    (dict(delta0=float("inf")), 1),
])
def test_fold_rejected(L, kw, code):
    p = fold_params(**kw)
    P = ctypes.c_void_p
    assert L.tri_fold_weights(ctypes.byref(p), P(FAKE), 4, P(FAKE), None) == code


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(tri, "_lib", None)
    monkeypatch.setattr(tri, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        tri.lib()


def test_score_max_checks(L):
    P = ctypes.c_void_p
    d = contig()                                   # packed [L][H][1][1000][128]
    assert L.tri_score_keys_max(ctypes.byref(d), P(FAKE), 65, P(FAKE), None) == 2     # too many offsets
    assert L.tri_score_keys_max(ctypes.byref(d), P(FAKE), 0, P(FAKE), None) == 1
    loose = contig(stride_head=1000 * 128 + 64, stride_layer=8 * (1000 * 128 + 64))
    assert L.tri_score_keys_max(ctypes.byref(loose), P(FAKE), 17, P(FAKE), None) == 2  # units not packed
    pg = paged(block_size=12, stride_block=12 * 4 * 128, stride_layer=100 * 12 * 4 * 128)
    assert L.tri_score_keys_max(ctypes.byref(pg), P(FAKE), 17, P(FAKE), None) == 2     # pages not a power of two
    # 8 heads x 32 weight columns exceed one MMA: one head per tile, and its pages are under 8 tokens
    pg = paged(num_kv_heads=8, block_size=4, stride_block=4 * 8 * 128, stride_layer=100 * 4 * 8 * 128,
               max_blocks_per_seq=16)
    assert L.tri_score_keys_max(ctypes.byref(pg), P(FAKE), 17, P(FAKE), None) == 2
    # a page of all 4 heads is 4 rows, under one 8-row swizzle atom
    pg = paged(block_size=1, stride_block=4 * 128, stride_layer=100 * 4 * 128, max_blocks_per_seq=64)
    assert L.tri_score_keys_max(ctypes.byref(pg), P(FAKE), 5, P(FAKE), None) == 2
    p = fold_params(offs=[1.0] * 3000)
    assert L.tri_fold_offset_weights(ctypes.byref(p), P(FAKE), 4, P(FAKE), None) == 2
    # the per-offset fold takes 32 centers per block along the grid's y (at most 65535 blocks)
    p = fold_params(offs=[1.0] * 2)
    assert L.tri_fold_offset_weights(ctypes.byref(p), P(FAKE), 65535 * 32 + 1, P(FAKE), None) == 2


def test_score_positions_checks(L):
    P = ctypes.c_void_p
    d = contig()
    fn = L.tri_score_keys_at_positions
    qp = (ctypes.c_int64 * 1)(5000)
    q = ctypes.cast(qp, P)
    assert fn(ctypes.byref(d), P(FAKE), 0.0, 0, None, q, P(FAKE), None) == 1             # theta
    assert fn(ctypes.byref(d), P(FAKE), float("inf"), 0, None, q, P(FAKE), None) == 1
    assert fn(ctypes.byref(d), P(FAKE), 1e4, 2, None, q, P(FAKE), None) == 1             # pairing
    assert fn(ctypes.byref(d), P(FAKE), 1e4, 0, None, None, P(FAKE), None) == 1          # no query positions
    assert fn(ctypes.byref(d), P(FAKE), 1e4, 0, P(FAKE + 2), q, P(FAKE), None) == 1      # misaligned positions
    for bad in (-1, 2 ** 31):
        qb = (ctypes.c_int64 * 1)(bad)
        assert fn(ctypes.byref(d), P(FAKE), 1e4, 0, None, ctypes.cast(qb, P), P(FAKE), None) == 1
    assert fn(ctypes.byref(contig(head_dim=64)), P(FAKE), 1e4, 0, None, q, P(FAKE), None) == 2


def test_binding_checks_buffers_before_the_library():
    """The C ABI takes plain pointers and cannot see a buffer's size: the
    binding checks each tensor before it calls the library; here a host tensor
    and a wrong dtype (short device buffers: test_gpu_parity)."""
    import torch
    k = torch.zeros((2, 3, 1, 16, 128), dtype=torch.bfloat16)
    d = tri.desc_contig(k, k)
    with pytest.raises(ValueError, match="w: need"):
        tri.score_keys(d, torch.zeros((6, 128)))                       # host memory
    with pytest.raises(ValueError, match="q_center: need"):
        tri.fold_weights(torch.zeros((6, 128), dtype=torch.float64), 1e4, [1.0])
