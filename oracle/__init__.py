"""CPU oracle (fp64) for the score -> select -> compact path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg are the only callers.  The product library never
imports, loads or calls anything here, and this package imports nothing from
the product.  The arithmetic lives in ``oracle.cpp`` (plain C++, fp64); this
module builds it with g++ and wraps it for numpy arrays.

Forms (all from the page "The future-offset average in TriAttention can be
precomputed"):

* ``score_cosine``   O-i   literal offset average of the cosine form
* ``score_literal``  O-ii  literal offset average of the complex form
* ``score_folded``   O-iii folded complex form with W_f
* ``score_polar``    O-iv  folded polar form with mu'_f = E[q_f] W_f
* ``score_max_literal``    the max-over-offsets variant, per offset literally
* ``score_at_positions``   the offset average at per-key distances (pre-RoPE cache)
* ``fold_w`` + ``score_realdot``  O-v  the real 2x2 per-band map, then a dot
* ``select``         keep-highest, ties to the lower index, ascending output
* ``gather_rows`` / ``holefill``  compaction, out of place / paged in place
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so next to it (plain g++, -O2, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.orc_frequencies.argtypes = [dbl, i32, P]
    lib.orc_offset_weights.argtypes = [dbl, i32, P, i32, P, P]
    for name in ("orc_score_cosine", "orc_score_literal", "orc_score_folded", "orc_score_polar",
                 "orc_score_max_literal"):
        getattr(lib, name).argtypes = [P, i64, i32, P, dbl, P, i32, dbl, i32, i32, P]
    lib.orc_score_at_positions.argtypes = [P, i64, i32, P, dbl, P, i32, P, i64, i32, i32, P]
    lib.orc_fold_w.argtypes = [P, i32, i32, dbl, P, i32, dbl, i32, P]
    lib.orc_score_realdot.argtypes = [P, i64, i32, P, i32, P]
    lib.orc_abs_dot.argtypes = [P, i64, i32, P, i32, P]
    lib.orc_select_f64.argtypes = [P, i64, i64, P]
    lib.orc_select_f64.restype = i64
    lib.orc_select_f32.argtypes = [P, i64, i64, P]
    lib.orc_select_f32.restype = i64
    lib.orc_gather_rows.argtypes = [P, i32, P, i64, P]
    lib.orc_holefill.argtypes = [P, i64, i32, P, i64, i64]
    lib.orc_holefill.restype = i64
    _lib = lib
    return lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _keys(keys) -> np.ndarray:
    """bf16 keys as their uint16 bit patterns, C-contiguous [n][d]."""
    try:
        import torch
        if isinstance(keys, torch.Tensor):
            assert keys.dtype == torch.bfloat16
            keys = keys.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(keys)
    assert a.dtype == np.uint16 and a.ndim == 2
    return a


def _vec(x, dtype) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def frequencies(theta: float, d: int) -> np.ndarray:
    out = np.empty(d // 2, dtype=np.float64)
    _load().orc_frequencies(theta, d, _ptr(out))
    return out


def offset_weights(theta: float, d: int, offsets: Sequence[float]) -> np.ndarray:
    """W_f as a complex128 array of length d/2."""
    D = _vec(offsets, np.float64)
    re = np.empty(d // 2)
    im = np.empty(d // 2)
    _load().orc_offset_weights(theta, d, _ptr(D), len(D), _ptr(re), _ptr(im))
    return re + 1j * im


def _score(fn, keys, qc, theta, offsets, delta0, pairing, threads):
    k = _keys(keys)
    q = _vec(qc, np.float32)
    D = _vec(offsets, np.float64)
    out = np.empty(k.shape[0], dtype=np.float64)
    fn(_ptr(k), k.shape[0], k.shape[1], _ptr(q), float(theta), _ptr(D), len(D),
       float(delta0), int(pairing), int(threads or default_threads()), _ptr(out))
    return out


def score_cosine(keys, qc, theta, offsets, delta0=0.0, pairing=0, threads=None):
    return _score(_load().orc_score_cosine, keys, qc, theta, offsets, delta0, pairing, threads)


def score_literal(keys, qc, theta, offsets, delta0=0.0, pairing=0, threads=None):
    return _score(_load().orc_score_literal, keys, qc, theta, offsets, delta0, pairing, threads)


def score_max_literal(keys, qc, theta, offsets, delta0=0.0, pairing=0, threads=None):
    """max over the schedule of the per-offset score (not foldable)."""
    return _score(_load().orc_score_max_literal, keys, qc, theta, offsets, delta0, pairing, threads)


def score_at_positions(keys, qc, theta, offsets, positions, t, pairing=0, threads=None):
    """Offset average at per-key distances t - positions[i] (pre-RoPE cache)."""
    k = _keys(keys)
    q = _vec(qc, np.float32)
    D = _vec(offsets, np.float64)
    pos = _vec(positions, np.int64)
    assert pos.shape[0] == k.shape[0]
    out = np.empty(k.shape[0], dtype=np.float64)
    _load().orc_score_at_positions(_ptr(k), k.shape[0], k.shape[1], _ptr(q), float(theta), _ptr(D), len(D),
                                   _ptr(pos), int(t), int(pairing), int(threads or default_threads()), _ptr(out))
    return out


def score_folded(keys, qc, theta, offsets, delta0=0.0, pairing=0, threads=None):
    return _score(_load().orc_score_folded, keys, qc, theta, offsets, delta0, pairing, threads)


def score_polar(keys, qc, theta, offsets, delta0=0.0, pairing=0, threads=None):
    return _score(_load().orc_score_polar, keys, qc, theta, offsets, delta0, pairing, threads)


def fold_w(centers, theta, offsets, delta0=0.0, pairing=0) -> np.ndarray:
    """fp64 real weight vectors [n][d] from fp32 centers [n][d] (the 2x2 map)."""
    q = _vec(centers, np.float32)
    q2 = q.reshape(-1, q.shape[-1])
    D = _vec(offsets, np.float64)
    out = np.empty(q2.shape, dtype=np.float64)
    _load().orc_fold_w(_ptr(q2), q2.shape[0], q2.shape[1], float(theta), _ptr(D), len(D),
                       float(delta0), int(pairing), _ptr(out))
    return out.reshape(q.shape)


def score_realdot(keys, w64, threads=None) -> np.ndarray:
    k = _keys(keys)
    w = _vec(w64, np.float64)
    out = np.empty(k.shape[0], dtype=np.float64)
    _load().orc_score_realdot(_ptr(k), k.shape[0], k.shape[1], _ptr(w),
                              int(threads or default_threads()), _ptr(out))
    return out


def abs_dot(keys, w64, threads=None) -> np.ndarray:
    """sum_j |w[j] k[j]| per key (the scale for the score tolerance)."""
    k = _keys(keys)
    w = _vec(w64, np.float64)
    out = np.empty(k.shape[0], dtype=np.float64)
    _load().orc_abs_dot(_ptr(k), k.shape[0], k.shape[1], _ptr(w),
                        int(threads or default_threads()), _ptr(out))
    return out


def select(scores, budget: int) -> np.ndarray:
    """Ascending indices of the top-min(B, n) scores (ties to the lower index,
    NaN lowest).  fp32 scores are ranked in fp32, fp64 in fp64."""
    try:
        import torch
        if isinstance(scores, torch.Tensor):
            scores = scores.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    s = np.ascontiguousarray(scores)
    n = s.shape[0]
    kept = np.empty(min(n, budget), dtype=np.int32)
    if s.dtype == np.float32:
        m = _load().orc_select_f32(_ptr(s), n, int(budget), _ptr(kept))
    else:
        s = s.astype(np.float64)
        m = _load().orc_select_f64(_ptr(s), n, int(budget), _ptr(kept))
    return kept[:m]


def gather_rows(rows, kept) -> np.ndarray:
    r = _keys(rows)
    k = _vec(kept, np.int32)
    out = np.empty((len(k), r.shape[1]), dtype=np.uint16)
    _load().orc_gather_rows(_ptr(r), r.shape[1], _ptr(k), len(k), _ptr(out))
    return out


def holefill(rows, kept, budget: int):
    """Return (rows after the in-place hole fill, number of rows moved)."""
    r = _keys(rows).copy()
    k = _vec(kept, np.int32)
    moved = _load().orc_holefill(_ptr(r), r.shape[0], r.shape[1], _ptr(k), len(k), int(budget))
    return r, int(moved)
