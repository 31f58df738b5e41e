"""Python binding of libdsa.so (the C ABI in include/dsa.h): argument marshalling only.

Every function here takes torch CUDA tensors, checks their dtype/shape/contiguity, and passes
raw device pointers, sizes and the current CUDA stream to the C entry point of the same name.
All computation runs in the library's CUDA kernels; there is no fallback of any kind: if the
library is missing this module raises at import time.

Shapes follow the C header:
  dsa_index(qI [Lq,HI,64], kI [Lk,64], w [Lq,HI], q_pos0, scores fp32 [Lq, ld])
  dsa_topk(scores fp32 [Lq, ld], q_pos0, k, idx int32 [Lq,k])
  dsa_sparse_attn(q [Lq,Hq,128], k/v [Lk,Hkv,128], idx [Lq,topk], q_pos0, scale, out, lse=None)
  dsa_prefill(q, k, v, qI, kI, w, topk, scale, out, idx_out=None, ws=None)
  dsa_decode(q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, topk, scale,
             out, idx_out=None, ws=None, update_ctx=False)
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "dsa.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -c 'import __graft_entry__ as g; g.build()'` "
                      "or `python dsa_lightning_indexer_02_b200/build.py` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_TIMEOUT, \
    DSA_ERR_DEVICE_INPUT = range(7)
DSA_OP_INDEX, DSA_OP_TOPK, DSA_OP_SPARSE_ATTN, DSA_OP_PREFILL, DSA_OP_DECODE, DSA_OP_INDEXER_KL = range(6)
PROFILE_KINDS = ("indexer", "topk", "sparse_attn", "combine", "decode_append", "advance", "selftest", "kl")

_p, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "dsa_status_string": (ctypes.c_char_p, [_i]),
    "dsa_version": (_i, []),
    "dsa_index": (_i, [_p, _p, _p, _i, _i64, _i, _i, _i64, _p, _i64, _p]),
    "dsa_topk": (_i, [_p, _i64, _i, _i64, _i, _p, _p, _sz, _p]),
    "dsa_topk_window": (_i, [_p, _i64, _i, _i64, _i, _i64, _p, _p]),
    "dsa_sparse_attn": (_i, [_p, _p, _p, _p, _i, _i64, _i64, _i, _i, _i, _i, _f, _p, _p, _p]),
    "dsa_prefill": (_i, [_p, _p, _p, _p, _p, _p, _i64, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _sz, _p]),
    "dsa_prefill_rows": (_i, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i, _i, _i, _i, _i, _i, _i64, _f, _p, _p, _p,
                              _sz, _p]),
    "dsa_prefill_window": (_i, [_p, _p, _p, _p, _p, _p, _i64, _i, _i, _i, _i, _i, _i, _i64, _f, _p, _p, _p, _sz,
                                _p]),
    "dsa_decode": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i64, _i, _i, _i, _i, _i, _i, _f, _i,
                        _p, _p, _p, _sz, _p]),
    "dsa_decode_noalloc": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i64, _i, _i, _i, _i, _i, _i, _f, _i,
                                _p, _p, _p]),
    "dsa_decode_noalloc_scratch_bytes": (_sz, []),
    "dsa_indexer_kl": (_i, [_p, _p, _p, _p, _p, _i64, _i, _i, _i, _i, _i, _f, _p, _p, _sz, _p]),
    "dsa_workspace_size": (_sz, [_i, _i64, _i, _i, _i, _i]),
    "dsa_sync_status": (_i, [_p]),
    "dsa_profile_begin": (None, []),
    "dsa_profile_end": (_i, [_p, _p]),
    "dsa_launch_count": (_i64, []),
    "dsa_read_counters": (_i, [_p, _i, _i]),
    "dsa_selftest_timeout": (_i, [_i64, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_symbols() -> list[str]:
    """Function names declared in include/dsa.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", text)))


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(status: int) -> str:
    return _lib.dsa_status_string(int(status)).decode()


def version() -> int:
    return int(_lib.dsa_version())


def _check(status: int, where: str) -> None:
    if status != DSA_OK:
        raise DSAError(status, where)


def _stream(stream=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")


def workspace_size(op: int, L: int, B: int = 1, Hq: int = 32, HI: int = 32, topk: int = 2048) -> int:
    return int(_lib.dsa_workspace_size(op, L, B, Hq, HI, topk))


def dsa_index(qI, kI, w, q_pos0: int, scores, stream=None) -> None:
    import torch
    _need(qI, torch.bfloat16, "qI", 3), _need(kI, torch.bfloat16, "kI", 2)
    _need(w, torch.bfloat16, "w", 2), _need(scores, torch.float32, "scores", 2)
    Lq, HI, dI = qI.shape
    st = _lib.dsa_index(_ptr(qI), _ptr(kI), _ptr(w), Lq, kI.shape[0], HI, dI, q_pos0, _ptr(scores),
                        scores.shape[1], _stream(stream))
    _check(st, "dsa_index")


def dsa_topk(scores, q_pos0: int, k: int, idx, window: int = 0, stream=None) -> None:
    import torch
    _need(scores, torch.float32, "scores", 2), _need(idx, torch.int32, "idx", 2)
    Lq = scores.shape[0]
    if idx.shape != (Lq, k):
        raise ValueError(f"idx must be [{Lq}, {k}]")
    if window:
        st = _lib.dsa_topk_window(_ptr(scores), scores.shape[1], Lq, q_pos0, k, window, _ptr(idx), _stream(stream))
        _check(st, "dsa_topk_window")
        return
    st = _lib.dsa_topk(_ptr(scores), scores.shape[1], Lq, q_pos0, k, _ptr(idx), None, 0, _stream(stream))
    _check(st, "dsa_topk")


def dsa_sparse_attn(q, k, v, idx, q_pos0: int, scale: float, out, lse=None, stream=None) -> None:
    import torch
    _need(q, torch.bfloat16, "q", 3), _need(k, torch.bfloat16, "k", 3), _need(v, torch.bfloat16, "v", 3)
    _need(idx, torch.int32, "idx", 2), _need(out, torch.bfloat16, "out", 3)
    if lse is not None:
        _need(lse, torch.float32, "lse", 2)
    Lq, Hq, D = q.shape
    if out.shape != q.shape or v.shape != k.shape or idx.shape[0] != Lq:
        raise ValueError("shape mismatch")
    st = _lib.dsa_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), Lq, k.shape[0], q_pos0, Hq, k.shape[1], D,
                              idx.shape[1], float(scale), _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "dsa_sparse_attn")


def dsa_prefill(q, k, v, qI, kI, w, topk: int, scale: float, out, idx_out=None, ws=None, window: int = 0,
                stream=None) -> None:
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (qI, "qI"), (out, "out")):
        _need(t, torch.bfloat16, n, 3)
    _need(kI, torch.bfloat16, "kI", 2), _need(w, torch.bfloat16, "w", 2)
    L, Hq, D = q.shape
    HI, dI = qI.shape[1], qI.shape[2]
    if ws is None:
        ws = torch.empty(workspace_size(DSA_OP_PREFILL, L, 1, Hq, HI, topk), dtype=torch.uint8, device=q.device)
    if idx_out is not None:
        _need(idx_out, torch.int32, "idx_out", 2)
    if window:
        st = _lib.dsa_prefill_window(_ptr(q), _ptr(k), _ptr(v), _ptr(qI), _ptr(kI), _ptr(w), L, Hq, k.shape[1], D,
                                     HI, dI, topk, window, float(scale), _ptr(out), _ptr(idx_out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream))
        _check(st, "dsa_prefill_window")
        return
    st = _lib.dsa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(qI), _ptr(kI), _ptr(w), L, Hq, k.shape[1], D, HI, dI,
                          topk, float(scale), _ptr(out), _ptr(idx_out), _ptr(ws), ws.numel() * ws.element_size(),
                          _stream(stream))
    _check(st, "dsa_prefill")


def dsa_prefill_rows(q_rows, k, v, qI_rows, kI, w_rows, row0: int, topk: int, scale: float, out_rows,
                     idx_rows=None, ws=None, window: int = 0, stream=None) -> None:
    """Prefill of query rows row0 .. row0+len(q_rows)-1; k, v, kI cover at least those rows."""
    import torch
    for t, n in ((q_rows, "q_rows"), (k, "k"), (v, "v"), (qI_rows, "qI_rows"), (out_rows, "out_rows")):
        _need(t, torch.bfloat16, n, 3)
    _need(kI, torch.bfloat16, "kI", 2), _need(w_rows, torch.bfloat16, "w_rows", 2)
    rows, Hq, D = q_rows.shape
    HI, dI = qI_rows.shape[1], qI_rows.shape[2]
    if k.shape[0] < row0 + rows or kI.shape[0] < row0 + rows:
        raise ValueError("k/v/kI must cover rows up to row0 + rows")
    if ws is None:
        ws = torch.empty(workspace_size(DSA_OP_PREFILL, row0 + rows, 1, Hq, HI, topk), dtype=torch.uint8,
                         device=q_rows.device)
    if idx_rows is not None:
        _need(idx_rows, torch.int32, "idx_rows", 2)
    st = _lib.dsa_prefill_rows(_ptr(q_rows), _ptr(k), _ptr(v), _ptr(qI_rows), _ptr(kI), _ptr(w_rows), row0, rows, Hq,
                               k.shape[1], D, HI, dI, topk, window, float(scale), _ptr(out_rows), _ptr(idx_rows),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "dsa_prefill_rows")


def dsa_indexer_kl(q, k, qI, kI, w, scale: float, kl, ws=None, stream=None) -> None:
    """Indexer warm-up target KL(P_t || Q_t) for every query row of one causal sequence into kl
    (float32 [L]); see dsa_indexer_kl in include/dsa.h."""
    import torch
    _need(q, torch.bfloat16, "q", 3), _need(k, torch.bfloat16, "k", 3), _need(qI, torch.bfloat16, "qI", 3)
    _need(kI, torch.bfloat16, "kI", 2), _need(w, torch.bfloat16, "w", 2), _need(kl, torch.float32, "kl", 1)
    L, Hq, D = q.shape
    HI, dI = qI.shape[1], qI.shape[2]
    if k.shape[0] < L or kI.shape[0] < L or kl.shape[0] < L:
        raise ValueError("k, kI and kl must cover the L query rows")
    if ws is None:
        ws = torch.empty(workspace_size(DSA_OP_INDEXER_KL, L, 1, Hq, HI, 1), dtype=torch.uint8, device=q.device)
    st = _lib.dsa_indexer_kl(_ptr(q), _ptr(k), _ptr(qI), _ptr(kI), _ptr(w), L, Hq, k.shape[1], D, HI, dI,
                             float(scale), _ptr(kl), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "dsa_indexer_kl")


def dsa_decode(q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, topk: int, scale: float, out,
               idx_out=None, ws=None, update_ctx: bool = False, stream=None) -> None:
    import torch
    for t, n in ((q, "q"), (qI, "qI"), (k_new, "k_new"), (v_new, "v_new"), (out, "out")):
        _need(t, torch.bfloat16, n, 3)
    _need(w, torch.bfloat16, "w", 2), _need(kI_new, torch.bfloat16, "kI_new", 2)
    _need(k_cache, torch.bfloat16, "k_cache", 4), _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(kI_cache, torch.bfloat16, "kI_cache", 3), _need(ctx_len, torch.int32, "ctx_len", 1)
    B, Hq, D = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    HI, dI = qI.shape[1], qI.shape[2]
    if ws is None:
        ws = torch.empty(workspace_size(DSA_OP_DECODE, Lmax, B, Hq, HI, topk), dtype=torch.uint8, device=q.device)
    if idx_out is not None:
        _need(idx_out, torch.int32, "idx_out", 2)
    st = _lib.dsa_decode(_ptr(q), _ptr(qI), _ptr(w), _ptr(k_new), _ptr(v_new), _ptr(kI_new), _ptr(k_cache),
                         _ptr(v_cache), _ptr(kI_cache), _ptr(ctx_len), B, Lmax, Hq, Hkv, D, HI, dI, topk,
                         float(scale), int(bool(update_ctx)), _ptr(out), _ptr(idx_out), _ptr(ws),
                         ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "dsa_decode")


def sync_status(stream=None) -> int:
    return int(_lib.dsa_sync_status(_stream(stream)))


def profile_begin() -> None:
    _lib.dsa_profile_begin()


def profile_end() -> dict:
    launches = (ctypes.c_int64 * len(PROFILE_KINDS))()
    ms = (ctypes.c_double * len(PROFILE_KINDS))()
    _check(_lib.dsa_profile_end(launches, ms), "dsa_profile_end")
    return {k: {"launches": int(launches[i]), "ms": float(ms[i])} for i, k in enumerate(PROFILE_KINDS)}


def read_counters(reset: bool = False) -> dict:
    """Device path counters: top-k rows and sampled-threshold fallbacks (see dsa.h)."""
    buf = (ctypes.c_int64 * 8)()
    _check(_lib.dsa_read_counters(buf, 8, int(bool(reset))), "dsa_read_counters")
    return {"topk_rows": buf[0], "topk_retry": buf[1], "topk_global": buf[4], "topk_cluster_rows": buf[2],
            "topk_cluster_retry": buf[3], "topk_cluster_global": buf[5]}


def launch_count() -> int:
    return int(_lib.dsa_launch_count())


def selftest_timeout(wait_ns: int, stream=None) -> None:
    _check(_lib.dsa_selftest_timeout(int(wait_ns), _stream(stream)), "dsa_selftest_timeout")


def lib() -> ctypes.CDLL:
    """The loaded C library (raw ctypes access for callers that marshal pointers themselves)."""
    return _lib
