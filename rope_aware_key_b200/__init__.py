"""Thin Python binding of libtri_evict.so (ctypes).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  If the
shared library is missing this module raises on import of the library (no
fallback of any kind).

    import rope_aware_key_b200 as tri
    d = tri.desc_contig(k, v)                 # k, v: bf16 [L][H][batch][N][128] on cuda
    w = tri.fold_weights(q_center, theta=1e6, offsets=[2.0**e for e in range(17)])
    kept, count = tri.compress(d, w, budget=2048, k_out=k_out, v_out=v_out)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "TriError", "lib", "Desc", "desc_contig", "desc_ragged", "desc_paged", "fold_weights", "score_keys",
    "select_topk", "compact_kv", "fold_offset_weights", "score_keys_max", "compress", "workspace_size",
    "score_row_stride", "read_device_status",
    "kernel_launches", "LAYOUT_CONTIG", "LAYOUT_RAGGED", "LAYOUT_PAGED", "PAIRING_HALF",
    "PAIRING_INTERLEAVED", "COMPACT_OUT_OF_PLACE", "COMPACT_IN_PLACE_HOLEFILL", "DEVFLAG_BAD_PAGE",
    "DEVFLAG_NONFINITE", "DEVFLAG_TIMEOUT", "DEVFLAG_BAD_KEPT", "DEVFLAG_BAD_POSITION", "DEVFLAG_INVARIANT",
    "load",
    "score_keys_at_positions",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtri_evict.so")

LAYOUT_CONTIG, LAYOUT_RAGGED, LAYOUT_PAGED = 0, 1, 2
PAIRING_HALF, PAIRING_INTERLEAVED = 0, 1
COMPACT_OUT_OF_PLACE, COMPACT_IN_PLACE_HOLEFILL = 0, 1
DEVFLAG_BAD_PAGE, DEVFLAG_NONFINITE, DEVFLAG_TIMEOUT, DEVFLAG_BAD_KEPT = 0x1, 0x2, 0x4, 0x8
DEVFLAG_BAD_POSITION = 0x10
DEVFLAG_INVARIANT = 0x20          # set only by a build with -DTRI_CHECKED
MAX_OFFSETS, MAX_BATCH, HEAD_DIM = 2048, 256, 128

_STATUS = {0: "TRI_OK", 1: "TRI_ERR_INVALID_ARG", 2: "TRI_ERR_UNSUPPORTED", 3: "TRI_ERR_WORKSPACE",
           4: "TRI_ERR_CUDA", 5: "TRI_ERR_DEVICE_CHECK", 6: "TRI_ERR_DEVICE_TIMEOUT"}


class TriError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        name = _STATUS.get(status, f"status {status}")
        extra = ""
        if status == 4:
            extra = f" (cudaError {lib().tri_last_cuda_error()})"
        super().__init__(f"{call}: {name}{extra}")


class _FoldParams(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("theta", ctypes.c_double),
                ("offsets", ctypes.POINTER(ctypes.c_double)), ("n_offsets", ctypes.c_int),
                ("delta0", ctypes.c_double), ("pairing", ctypes.c_int)]


class _CacheDesc(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int), ("num_layers", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("batch", ctypes.c_int), ("max_seq_len", ctypes.c_int),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("stride_layer", ctypes.c_int64), ("stride_head", ctypes.c_int64),
                ("stride_seq", ctypes.c_int64), ("stride_block", ctypes.c_int64),
                ("seq_len", ctypes.c_int),
                ("cu_seqlens", ctypes.POINTER(ctypes.c_int32)), ("seq_lens", ctypes.POINTER(ctypes.c_int32)),
                ("block_table", ctypes.c_void_p), ("max_blocks_per_seq", ctypes.c_int),
                ("block_size", ctypes.c_int), ("num_blocks", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m rope_aware_key_b200.build` "
                          "(there is no fallback implementation)")
    _lib = load(LIB_PATH)
    return _lib


def load(path: str) -> ctypes.CDLL:
    """A build of the library at `path` with the call signatures set (the
    product library, or one of the test-only builds of the same sources)."""
    L = ctypes.CDLL(path)
    P, I, I64, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    D = ctypes.POINTER(_CacheDesc)
    L.tri_fold_weights.argtypes = [ctypes.POINTER(_FoldParams), P, I, P, P]
    L.tri_fold_offset_weights.argtypes = [ctypes.POINTER(_FoldParams), P, I, P, P]
    L.tri_score_keys_max.argtypes = [D, P, I, P, P]
    L.tri_score_keys_at_positions.argtypes = [D, P, ctypes.c_double, I, P, P, P, P]
    L.tri_score_row_stride.argtypes = [D]
    L.tri_score_row_stride.restype = I64
    L.tri_score_keys.argtypes = [D, P, P, P]
    L.tri_select_topk.argtypes = [D, P, I, P, P, P]
    L.tri_compact_kv.argtypes = [D, P, P, I, I, P, P, P]
    L.tri_workspace_size.argtypes = [D, I, ctypes.POINTER(S)]
    L.tri_compress.argtypes = [D, P, I, I, P, P, P, P, P, S, P]
    L.tri_compress_max.argtypes = [D, P, I, I, I, P, P, P, P, P, S, P]
    L.tri_read_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), I]
    L.tri_status_string.argtypes = [I]
    L.tri_status_string.restype = ctypes.c_char_p
    L.tri_last_cuda_error.restype = I
    L.tri_kernel_launches.restype = ctypes.c_uint64
    L.tri_version.restype = ctypes.c_char_p
    for name in ("tri_fold_weights", "tri_fold_offset_weights", "tri_score_keys_max", "tri_score_keys",
                 "tri_score_keys_at_positions", "tri_select_topk", "tri_compact_kv", "tri_workspace_size",
                 "tri_compress", "tri_compress_max", "tri_read_device_status"):
        getattr(L, name).restype = I
    return L


def _check(st: int, call: str) -> None:
    if st != 0:
        raise TriError(st, call)


def _stream(stream, device=None) -> ctypes.c_void_p:
    """The given stream, or the current stream of `device` (the device that
    holds the call's tensors: the library launches there)."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t: Optional[torch.Tensor], dtype: torch.dtype, numel: int, name: str) -> None:
    """The library takes plain pointers and cannot see a buffer's size, so the
    binding checks each tensor it passes: device memory of the right type,
    contiguous, and at least as many elements as the call touches."""
    if t is None:
        return
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous() and t.numel() >= numel):
        raise ValueError(f"{name}: need a contiguous {dtype} cuda tensor of >= {numel} elements, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}" + ("" if t.is_contiguous() else " (strided)"))


class Desc:
    """A tri_cache_desc plus the host arrays and tensors it points to."""

    def __init__(self, raw: _CacheDesc, keep: list, units: int, lens: Sequence[int]):
        self.raw = raw
        self._keep = keep
        self.units = units
        self.lens = list(lens)

    @property
    def ref(self):
        return ctypes.byref(self.raw)

    @property
    def num_layers(self):
        return self.raw.num_layers

    @property
    def num_kv_heads(self):
        return self.raw.num_kv_heads

    @property
    def batch(self):
        return self.raw.batch


def _i32_host(values) -> ctypes.Array:
    vals = [int(x) for x in values]
    return (ctypes.c_int32 * len(vals))(*vals)


def desc_contig(k: torch.Tensor, v: Optional[torch.Tensor] = None, max_seq_len: int = 0) -> Desc:
    """k, v: bf16 [L][H][batch][N][128] with the last two dims packed.  k on
    the device; v on the same device, or a pinned CPU tensor for out-of-place
    compaction (the gather reads only the kept rows over the bus)."""
    assert k.dim() == 5 and k.dtype == torch.bfloat16 and k.shape[-1] == HEAD_DIM
    assert k.stride(-1) == 1 and k.stride(-2) == HEAD_DIM
    if v is not None:
        assert v.shape == k.shape and v.stride() == k.stride() and v.dtype == k.dtype
    L, H, Bt, N, _ = k.shape
    raw = _CacheDesc(layout=LAYOUT_CONTIG, num_layers=L, num_kv_heads=H, head_dim=HEAD_DIM, batch=Bt,
                     max_seq_len=max_seq_len, k=k.data_ptr(), v=v.data_ptr() if v is not None else None,
                     stride_layer=k.stride(0), stride_head=k.stride(1), stride_seq=k.stride(2), seq_len=N)
    return Desc(raw, [k, v], L * H * Bt, [N] * Bt)


def desc_ragged(k: torch.Tensor, v: Optional[torch.Tensor], cu_seqlens: Sequence[int],
                max_seq_len: int = 0) -> Desc:
    """k, v: bf16 [L][H][T][128]; cu_seqlens: host ints [batch+1]."""
    assert k.dim() == 4 and k.dtype == torch.bfloat16 and k.stride(-1) == 1 and k.stride(-2) == HEAD_DIM
    if v is not None:
        assert v.shape == k.shape and v.stride() == k.stride()
    cu = [int(x) for x in (cu_seqlens.tolist() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens)]
    L, H = k.shape[0], k.shape[1]
    Bt = len(cu) - 1
    cu_arr = _i32_host(cu)
    raw = _CacheDesc(layout=LAYOUT_RAGGED, num_layers=L, num_kv_heads=H, head_dim=HEAD_DIM, batch=Bt,
                     max_seq_len=max_seq_len, k=k.data_ptr(), v=v.data_ptr() if v is not None else None,
                     stride_layer=k.stride(0), stride_head=k.stride(1),
                     cu_seqlens=ctypes.cast(cu_arr, ctypes.POINTER(ctypes.c_int32)))
    lens = [cu[i + 1] - cu[i] for i in range(Bt)]
    return Desc(raw, [k, v, cu_arr], L * H * Bt, lens)


def desc_paged(k: torch.Tensor, v: Optional[torch.Tensor], block_table: torch.Tensor,
               seq_lens: Sequence[int], max_seq_len: int = 0) -> Desc:
    """k, v: bf16 [L][num_blocks][block_size][H][128] (pages packed);
    block_table: int32 cuda [batch][max_blocks]; seq_lens: host ints [batch]."""
    assert k.dim() == 5 and k.dtype == torch.bfloat16 and k.shape[-1] == HEAD_DIM
    assert k.stride(-1) == 1 and k.stride(-2) == HEAD_DIM and k.stride(-3) == HEAD_DIM * k.shape[3]
    assert block_table.dtype == torch.int32 and block_table.is_cuda and block_table.is_contiguous()
    if v is not None:
        assert v.shape == k.shape and v.stride() == k.stride()
    L, NB, bs, H, _ = k.shape
    lens = [int(x) for x in (seq_lens.tolist() if isinstance(seq_lens, torch.Tensor) else seq_lens)]
    lens_arr = _i32_host(lens)
    raw = _CacheDesc(layout=LAYOUT_PAGED, num_layers=L, num_kv_heads=H, head_dim=HEAD_DIM, batch=len(lens),
                     max_seq_len=max_seq_len, k=k.data_ptr(), v=v.data_ptr() if v is not None else None,
                     stride_layer=k.stride(0), stride_block=k.stride(1),
                     seq_lens=ctypes.cast(lens_arr, ctypes.POINTER(ctypes.c_int32)),
                     block_table=block_table.data_ptr(), max_blocks_per_seq=block_table.shape[1],
                     block_size=bs, num_blocks=NB)
    return Desc(raw, [k, v, block_table, lens_arr], L * H * len(lens), lens)


def fold_weights(q_center: torch.Tensor, theta: float, offsets: Sequence[float], delta0: float = 0.0,
                 pairing: int = PAIRING_HALF, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Fold the offset average into fp32 weights [n][128] (on the device)."""
    q = q_center.reshape(-1, HEAD_DIM)
    _need(q, torch.float32, q.numel(), "q_center")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.float32, q.numel(), "out")
    offs = [float(x) for x in offsets]
    arr = (ctypes.c_double * len(offs))(*offs)
    p = _FoldParams(head_dim=HEAD_DIM, theta=float(theta), offsets=arr, n_offsets=len(offs),
                    delta0=float(delta0), pairing=int(pairing))
    _check(lib().tri_fold_weights(ctypes.byref(p), _ptr(q), q.shape[0], _ptr(out), _stream(stream, q.device)),
           "tri_fold_weights")
    return out


def fold_offset_weights(q_center: torch.Tensor, theta: float, offsets: Sequence[float], delta0: float = 0.0,
                        pairing: int = PAIRING_HALF, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """Per-offset (unaveraged) weights, fp32 [n][len(offsets)][128] on the device."""
    q = q_center.reshape(-1, HEAD_DIM)
    _need(q, torch.float32, q.numel(), "q_center")
    offs = [float(x) for x in offsets]
    if out is None:
        out = torch.empty((q.shape[0], len(offs), HEAD_DIM), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, q.numel() * len(offs), "out")
    arr = (ctypes.c_double * len(offs))(*offs)
    p = _FoldParams(head_dim=HEAD_DIM, theta=float(theta), offsets=arr, n_offsets=len(offs),
                    delta0=float(delta0), pairing=int(pairing))
    _check(lib().tri_fold_offset_weights(ctypes.byref(p), _ptr(q), q.shape[0], _ptr(out),
                                         _stream(stream, q.device)),
           "tri_fold_offset_weights")
    return out


def score_keys_max(d: Desc, w_offsets: torch.Tensor, scores: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Max over the offsets of the per-offset scores (tensor cores)."""
    n_off = w_offsets.shape[-2]
    _need(w_offsets, torch.float32, d.num_layers * d.num_kv_heads * n_off * HEAD_DIM, "w_offsets")
    if scores is None:
        scores = torch.empty((d.units, score_row_stride(d)), dtype=torch.float32, device=w_offsets.device)
    _need(scores, torch.float32, d.units * score_row_stride(d), "scores")
    _check(lib().tri_score_keys_max(d.ref, _ptr(w_offsets), int(n_off), _ptr(scores),
                                    _stream(stream, w_offsets.device)),
           "tri_score_keys_max")
    return scores


def score_row_stride(d: Desc) -> int:
    s = lib().tri_score_row_stride(d.ref)
    if s < 0:
        raise TriError(1, "tri_score_row_stride")
    return int(s)


def score_keys(d: Desc, w: torch.Tensor, scores: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need(w, torch.float32, d.num_layers * d.num_kv_heads * HEAD_DIM, "w")
    if scores is None:
        scores = torch.empty((d.units, score_row_stride(d)), dtype=torch.float32, device=w.device)
    _need(scores, torch.float32, d.units * score_row_stride(d), "scores")
    _check(lib().tri_score_keys(d.ref, _ptr(w), _ptr(scores), _stream(stream, w.device)), "tri_score_keys")
    return scores


def score_keys_at_positions(d: Desc, w: torch.Tensor, theta: float, query_pos: Sequence[int],
                            positions: Optional[torch.Tensor] = None, pairing: int = PAIRING_HALF,
                            scores: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Offset-averaged score of a pre-RoPE cache at each key's own distance
    t_b - p_i.  positions: device int32 laid out like the scores, or None for
    p_i = i; query_pos: one position per sequence."""
    stride = score_row_stride(d)
    _need(w, torch.float32, d.num_layers * d.num_kv_heads * HEAD_DIM, "w")
    if scores is None:
        scores = torch.empty((d.units, stride), dtype=torch.float32, device=w.device)
    _need(scores, torch.float32, d.units * stride, "scores")
    _need(positions, torch.int32, d.units * stride, "positions")
    if len(query_pos) < d.batch:
        raise ValueError(f"query_pos: need one position per sequence ({d.batch}), got {len(query_pos)}")
    qp = (ctypes.c_int64 * max(1, len(query_pos)))(*[int(t) for t in query_pos])
    _check(lib().tri_score_keys_at_positions(d.ref, _ptr(w), float(theta), int(pairing), _ptr(positions),
                                             ctypes.cast(qp, ctypes.c_void_p), _ptr(scores),
                                             _stream(stream, w.device)),
           "tri_score_keys_at_positions")
    return scores


def select_topk(d: Desc, scores: torch.Tensor, budget: int, kept: Optional[torch.Tensor] = None,
                kept_count: Optional[torch.Tensor] = None, stream=None):
    _need(scores, torch.float32, d.units * score_row_stride(d), "scores")
    if kept is None:
        kept = torch.empty((d.units, budget), dtype=torch.int32, device=scores.device)
    if kept_count is None:
        kept_count = torch.empty((d.units,), dtype=torch.int32, device=scores.device)
    _need(kept, torch.int32, d.units * max(int(budget), 0), "kept")
    _need(kept_count, torch.int32, d.units, "kept_count")
    _check(lib().tri_select_topk(d.ref, _ptr(scores), int(budget), _ptr(kept), _ptr(kept_count),
                                 _stream(stream, scores.device)),
           "tri_select_topk")
    return kept, kept_count


def compact_kv(d: Desc, kept: torch.Tensor, kept_count: torch.Tensor, budget: int,
               mode: int = COMPACT_OUT_OF_PLACE, k_out: Optional[torch.Tensor] = None,
               v_out: Optional[torch.Tensor] = None, stream=None) -> None:
    _need(kept, torch.int32, d.units * max(int(budget), 0), "kept")
    _need(kept_count, torch.int32, d.units, "kept_count")
    _need(k_out, torch.bfloat16, d.units * max(int(budget), 0) * HEAD_DIM, "k_out")
    _need(v_out, torch.bfloat16, d.units * max(int(budget), 0) * HEAD_DIM, "v_out")
    _check(lib().tri_compact_kv(d.ref, _ptr(kept), _ptr(kept_count), int(budget), int(mode), _ptr(k_out),
                                _ptr(v_out), _stream(stream, kept.device)), "tri_compact_kv")


def workspace_size(d: Desc, budget: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tri_workspace_size(d.ref, int(budget), ctypes.byref(n)), "tri_workspace_size")
    return int(n.value)


def compress(d: Desc, w: torch.Tensor, budget: int, mode: int = COMPACT_OUT_OF_PLACE,
             kept: Optional[torch.Tensor] = None, kept_count: Optional[torch.Tensor] = None,
             k_out: Optional[torch.Tensor] = None, v_out: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, stream=None):
    """score -> select -> compact; returns (kept, kept_count)."""
    dev = w.device
    if kept is None:
        kept = torch.empty((d.units, budget), dtype=torch.int32, device=dev)
    if kept_count is None:
        kept_count = torch.empty((d.units,), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(workspace_size(d, budget), dtype=torch.uint8, device=dev)
    nb = d.units * max(int(budget), 0)
    _need(w, torch.float32, d.num_layers * d.num_kv_heads * HEAD_DIM, "w")
    _need(kept, torch.int32, nb, "kept")
    _need(kept_count, torch.int32, d.units, "kept_count")
    _need(k_out, torch.bfloat16, nb * HEAD_DIM, "k_out")
    _need(v_out, torch.bfloat16, nb * HEAD_DIM, "v_out")
    _need(workspace, torch.uint8, 0, "workspace")      # its size goes to the library, which checks it
    _check(lib().tri_compress(d.ref, _ptr(w), int(budget), int(mode), _ptr(kept), _ptr(kept_count), _ptr(k_out),
                              _ptr(v_out), _ptr(workspace), workspace.numel(), _stream(stream, dev)),
           "tri_compress")
    return kept, kept_count


def compress_max(d: Desc, w_offsets: torch.Tensor, budget: int, mode: int = COMPACT_OUT_OF_PLACE,
                 kept: Optional[torch.Tensor] = None, kept_count: Optional[torch.Tensor] = None,
                 k_out: Optional[torch.Tensor] = None, v_out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """max-over-offsets score -> select -> compact; returns (kept, kept_count)."""
    dev = w_offsets.device
    n_off = w_offsets.shape[-2]
    if kept is None:
        kept = torch.empty((d.units, budget), dtype=torch.int32, device=dev)
    if kept_count is None:
        kept_count = torch.empty((d.units,), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(workspace_size(d, budget), dtype=torch.uint8, device=dev)
    nb = d.units * max(int(budget), 0)
    _need(w_offsets, torch.float32, d.num_layers * d.num_kv_heads * n_off * HEAD_DIM, "w_offsets")
    _need(kept, torch.int32, nb, "kept")
    _need(kept_count, torch.int32, d.units, "kept_count")
    _need(k_out, torch.bfloat16, nb * HEAD_DIM, "k_out")
    _need(v_out, torch.bfloat16, nb * HEAD_DIM, "v_out")
    _need(workspace, torch.uint8, 0, "workspace")      # its size goes to the library, which checks it
    _check(lib().tri_compress_max(d.ref, _ptr(w_offsets), int(n_off), int(budget), int(mode), _ptr(kept),
                                  _ptr(kept_count), _ptr(k_out), _ptr(v_out), _ptr(workspace), workspace.numel(),
                                  _stream(stream, dev)),
           "tri_compress_max")
    return kept, kept_count


def read_device_status(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return the device status bits (DEVFLAG_*)."""
    flags = ctypes.c_uint32(0)
    st = lib().tri_read_device_status(_stream(stream), ctypes.byref(flags), int(bool(clear)))
    if st not in (0, 5, 6):
        raise TriError(st, "tri_read_device_status")
    return int(flags.value)


def kernel_launches() -> int:
    return int(lib().tri_kernel_launches())
