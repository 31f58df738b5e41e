"""DSA oracle -- TEST INFRASTRUCTURE ONLY.

Python access (ctypes) to the plain fp64 C oracle in oracle.c.  Only the tests, the package's
smoke check and the benchmark's CPU-baseline leg may import this module; the library path never
does, and the two share no code.  See oracle.c for what each step computes and which page
passage it follows.

All tensor inputs are numpy uint16 arrays holding bf16 bit patterns, laid out as the CUDA
library's inputs: q [rows, Hq, D], k/v [Lk, Hkv, D], qI [rows, HI, dI], kI [Lk, dI], w [rows, HI].
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", src, "-o", _SO, "-lm"])
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        p, i64, i32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_index_rows.argtypes = [p, p, p, p, i64, i32, i32, p, i64]
        lib.oracle_topk_rows.argtypes = [p, i64, p, p, i64, i32, p, p]
        lib.oracle_sparse_attn_rows.argtypes = [p, p, p, p, i64, i32, i32, i32, i32, f64, p, p]
        lib.oracle_dsa_rows.argtypes = [p, p, p, p, p, p, p, i64, i32, i32, i32, i32, i32, i32, i64, f64,
                                        p, p, p, p, i64, p, p]
        lib.oracle_kl_rows.argtypes = [p, p, p, p, p, p, i64, i32, i32, i32, i32, i32, f64, p]
        lib.oracle_num_threads.restype = i32
        for f in ("oracle_index_rows", "oracle_topk_rows", "oracle_sparse_attn_rows",
                  "oracle_dsa_rows", "oracle_kl_rows"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


def threads() -> int:
    return int(_load().oracle_num_threads())


def index_rows(qI: np.ndarray, w: np.ndarray, kI: np.ndarray, t_rows) -> np.ndarray:
    """Indexer scores, float64 [rows, max t + 1]; entries s > t are NaN."""
    t_rows = _c(np.atleast_1d(t_rows), np.int64)
    nr = t_rows.size
    HI, dI = qI.shape[-2], qI.shape[-1]
    qI, w, kI = _c(qI, np.uint16), _c(w, np.uint16), _c(kI, np.uint16)
    assert qI.shape[0] == nr and w.shape == (nr, HI) and kI.shape[1] == dI
    assert kI.shape[0] >= int(t_rows.max()) + 1
    ld = int(t_rows.max()) + 1
    scores = np.full((nr, ld), np.nan)
    _load().oracle_index_rows(_ptr(qI), _ptr(w), _ptr(kI), _ptr(t_rows), nr, HI, dI, _ptr(scores), ld)
    return scores


def topk_rows(scores: np.ndarray, n_valid, k: int, window: int = 0):
    """(idx int32 [rows, k] ordered by (score desc, index asc), -1 padded; tau float64 [rows]).

    With window > 0 only keys n-window .. n-1 of a row with n valid keys compete."""
    scores = _c(scores, np.float64)
    n_valid = _c(np.atleast_1d(n_valid), np.int64)
    nr, ld = scores.shape
    assert n_valid.size == nr and int(n_valid.max(initial=0)) <= ld
    first = None
    if window > 0:
        first = _c(np.maximum(0, n_valid - window), np.int64)
    idx = np.empty((nr, k), dtype=np.int32)
    tau = np.empty(nr)
    _load().oracle_topk_rows(_ptr(scores), ld, _ptr(n_valid), _ptr(first), nr, k, _ptr(idx), _ptr(tau))
    return idx, tau


def sparse_attn_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, idx: np.ndarray, scale: float):
    """(out float64 [rows, Hq, D], lse float64 [rows, Hq]) over the keys listed in idx."""
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    idx = _c(idx, np.int32)
    nr, Hq, D = q.shape
    Hkv = k.shape[1]
    assert k.shape[2] == D and v.shape == k.shape and idx.shape[0] == nr
    assert Hq % Hkv == 0
    if idx.size:
        assert int(idx.max()) < k.shape[0]
    topk = idx.shape[1]
    out = np.empty((nr, Hq, D))
    lse = np.empty((nr, Hq))
    _load().oracle_sparse_attn_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), nr, topk, Hq, Hkv, D,
                                    float(scale), _ptr(out), _ptr(lse))
    return out, lse


def dsa_rows(q_rows, qI_rows, w_rows, k, v, kI, t_rows, topk: int, scale: float,
             keep_scores: bool = False, window: int = 0) -> dict:
    """All three steps for query positions t_rows of one causal sequence.

    q_rows/qI_rows/w_rows hold the rows of those positions only; k, v, kI hold the whole prefix.
    Returns idx, out, lse, tau (score of the last selected key), absmax (max |score| of the row)
    and, with keep_scores, the score rows (NaN beyond t).  window > 0: sliding-window top-k over
    keys t-window+1 .. t (the scores and absmax still cover the whole causal row).
    """
    t_rows = _c(np.atleast_1d(t_rows), np.int64)
    nr = t_rows.size
    q_rows, qI_rows, w_rows = _c(q_rows, np.uint16), _c(qI_rows, np.uint16), _c(w_rows, np.uint16)
    k, v, kI = _c(k, np.uint16), _c(v, np.uint16), _c(kI, np.uint16)
    _, Hq, D = q_rows.shape
    Hkv = k.shape[1]
    HI, dI = qI_rows.shape[1], qI_rows.shape[2]
    assert q_rows.shape[0] == nr and qI_rows.shape[0] == nr and w_rows.shape == (nr, HI)
    assert k.shape[0] >= int(t_rows.max()) + 1 and kI.shape[0] >= int(t_rows.max()) + 1
    idx = np.empty((nr, topk), dtype=np.int32)
    out = np.empty((nr, Hq, D))
    lse = np.empty((nr, Hq))
    tau = np.empty(nr)
    absmax = np.empty(nr)
    ld = int(t_rows.max()) + 1
    scores = np.full((nr, ld), np.nan) if keep_scores else None
    _load().oracle_dsa_rows(_ptr(q_rows), _ptr(qI_rows), _ptr(w_rows), _ptr(k), _ptr(v), _ptr(kI),
                            _ptr(t_rows), nr, Hq, Hkv, D, HI, dI, topk, int(window), float(scale), _ptr(idx),
                            _ptr(out), _ptr(lse), _ptr(scores), ld, _ptr(tau), _ptr(absmax))
    res = {"idx": idx, "out": out, "lse": lse, "tau": tau, "absmax": absmax}
    if keep_scores:
        res["scores"] = scores
    return res


def kl_rows(q_rows, k, qI_rows, w_rows, kI, t_rows, scale: float) -> np.ndarray:
    """Indexer warm-up target KL(P_t || Q_t) (float64 [rows]) for query positions t_rows: P_t the
    dense causal attention distribution averaged over the Hq heads, Q_t the softmax of the
    indexer scores over keys 0..t.  q_rows/qI_rows/w_rows hold those positions' rows; k and kI
    the whole prefix."""
    t_rows = _c(np.atleast_1d(t_rows), np.int64)
    nr = t_rows.size
    q_rows, qI_rows, w_rows = _c(q_rows, np.uint16), _c(qI_rows, np.uint16), _c(w_rows, np.uint16)
    k, kI = _c(k, np.uint16), _c(kI, np.uint16)
    _, Hq, D = q_rows.shape
    Hkv = k.shape[1]
    HI, dI = qI_rows.shape[1], qI_rows.shape[2]
    assert q_rows.shape[0] == nr and qI_rows.shape[0] == nr and w_rows.shape == (nr, HI)
    assert Hq % Hkv == 0 and k.shape[2] == D and kI.shape[1] == dI
    assert k.shape[0] >= int(t_rows.max()) + 1 and kI.shape[0] >= int(t_rows.max()) + 1
    kl = np.empty(nr)
    _load().oracle_kl_rows(_ptr(q_rows), _ptr(k), _ptr(qI_rows), _ptr(w_rows), _ptr(kI), _ptr(t_rows), nr, Hq, Hkv,
                           D, HI, dI, float(scale), _ptr(kl))
    return kl
