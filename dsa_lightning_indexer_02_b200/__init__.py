"""Python binding of libdsa.so (the C ABI in include/dsa.h): argument marshalling only.

Every function here takes torch CUDA tensors, checks their dtype/shape/contiguity, and passes
raw device pointers, sizes and the current CUDA stream to the C entry point of the same name.
All computation runs in the library's CUDA kernels; there is no fallback of any kind: if the
library is missing this module raises at import time.

Shapes follow the C header (bf16 unless stated; every shape is checked before the call):
  dsa_index(qI [Lq,HI,64], kI [Lk,64], w [Lq,HI], q_pos0, scores fp32 [Lq, ld])
  dsa_topk(scores fp32 [Lq, ld], q_pos0, k, idx int32 [Lq,k], window=0)
  dsa_sparse_attn(q [Lq,Hq,128], k/v [Lk,Hkv,128], idx int32 [Lq,topk], q_pos0, scale, out [Lq,Hq,128],
                  lse fp32 [Lq,Hq] = None)
  dsa_prefill(q [L,Hq,128], k/v [>=L,Hkv,128], qI [L,HI,64], kI [>=L,64], w [L,HI], topk, scale,
              out [L,Hq,128], idx_out int32 [L,topk] = None, ws=None, window=0)
  dsa_prefill_rows(q_rows [R,..], k, v, qI_rows [R,..], kI, w_rows [R,HI], row0, topk, scale, out_rows,
                   idx_rows=None, ws=None, window=0)      (k/v/kI cover rows 0 .. row0+R-1)
  dsa_indexer_kl(q [L,Hq,128], k [>=L,Hkv,128], qI [L,HI,64], kI [>=L,64], w [L,HI], scale, kl fp32 [>=L])
  dsa_decode(q [B,Hq,128], qI [B,HI,64], w [B,HI], k_new/v_new [B,Hkv,128], kI_new [B,64],
             k_cache/v_cache [B,Lmax,Hkv,128], kI_cache [B,Lmax,64], ctx_len int32 [B], topk, scale,
             out [B,Hq,128], idx_out int32 [B,topk] = None, ws=None, update_ctx=False)
Every tensor must be contiguous and on the current CUDA device.
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
    "dsa_sparse_attn_dedup": (_i, [_p, _p, _p, _p, _i, _i64, _i64, _i, _i, _i, _i, _f, _p, _p, _p]),
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
    "dsa_error_site": (ctypes.c_uint, []),
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


def _need(t, dtype, name, shape):
    """One tensor argument: its type, dtype, shape (None: any extent) and contiguity.  The
    library reads every size from the leading operand, so an operand whose shape disagrees would
    let a kernel read or write past it: refuse it here."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != len(shape) or any(e is not None and int(e) != n for e, n in zip(shape, t.shape)):
        want = ", ".join("*" if e is None else str(int(e)) for e in shape)
        raise ValueError(f"{name} must have shape [{want}], got {list(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _at_least(t, name, dim, n):
    if t.shape[dim] < n:
        raise ValueError(f"{name}.shape[{dim}] must be >= {n}, got {t.shape[dim]}")


def _on_device(**tensors):
    """Every tensor argument on the current CUDA device (where the library launches)."""
    import torch
    ts = {k: t for k, t in tensors.items() if t is not None}
    for k, t in ts.items():
        if not t.is_cuda:
            raise ValueError(f"{k} must be a CUDA tensor")
    dev = torch.cuda.current_device()
    for k, t in ts.items():
        if t.device.index != dev:
            raise ValueError(f"{k} is on {t.device}, the current device is cuda:{dev}")


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def workspace_size(op: int, L: int, B: int = 1, Hq: int = 32, HI: int = 32, topk: int = 2048) -> int:
    return int(_lib.dsa_workspace_size(op, L, B, Hq, HI, topk))


def _workspace(ws, op, L, B, Hq, HI, topk, like):
    import torch
    if ws is None:
        return torch.empty(workspace_size(op, L, B, Hq, HI, topk), dtype=torch.uint8, device=like.device)
    if not isinstance(ws, torch.Tensor) or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous torch.Tensor")
    return ws


def dsa_index(qI, kI, w, q_pos0: int, scores, stream=None) -> None:
    """scores[i, s] for the Lq rows of qI (positions q_pos0 + i) and every causal key s."""
    import torch
    bf = torch.bfloat16
    _need(qI, bf, "qI", (None, None, None))
    Lq, HI, dI = qI.shape
    _need(kI, bf, "kI", (None, dI)), _need(w, bf, "w", (Lq, HI)), _need(scores, torch.float32, "scores", (Lq, None))
    _on_device(qI=qI, kI=kI, w=w, scores=scores)
    st = _lib.dsa_index(_ptr(qI), _ptr(kI), _ptr(w), Lq, kI.shape[0], HI, dI, q_pos0, _ptr(scores),
                        scores.shape[1], _stream(stream))
    _check(st, "dsa_index")


def dsa_topk(scores, q_pos0: int, k: int, idx, window: int = 0, stream=None) -> None:
    """idx[i] = the top-k keys of score row i (row i holds q_pos0 + i + 1 valid scores)."""
    import torch
    _need(scores, torch.float32, "scores", (None, None))
    Lq = scores.shape[0]
    _need(idx, torch.int32, "idx", (Lq, k))
    _on_device(scores=scores, idx=idx)
    if window:
        st = _lib.dsa_topk_window(_ptr(scores), scores.shape[1], Lq, q_pos0, k, window, _ptr(idx), _stream(stream))
        _check(st, "dsa_topk_window")
        return
    st = _lib.dsa_topk(_ptr(scores), scores.shape[1], Lq, q_pos0, k, _ptr(idx), None, 0, _stream(stream))
    _check(st, "dsa_topk")


def dsa_sparse_attn(q, k, v, idx, q_pos0: int, scale: float, out, lse=None, stream=None) -> None:
    """Attention of the Lq rows of q over the keys that idx selects for each row."""
    import torch
    bf = torch.bfloat16
    _need(q, bf, "q", (None, None, None))
    Lq, Hq, D = q.shape
    _need(k, bf, "k", (None, None, D))
    _need(v, bf, "v", tuple(k.shape)), _need(idx, torch.int32, "idx", (Lq, None)), _need(out, bf, "out", (Lq, Hq, D))
    if lse is not None:
        _need(lse, torch.float32, "lse", (Lq, Hq))
    _on_device(q=q, k=k, v=v, idx=idx, out=out, lse=lse)
    st = _lib.dsa_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), Lq, k.shape[0], q_pos0, Hq, k.shape[1], D,
                              idx.shape[1], float(scale), _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "dsa_sparse_attn")


def dsa_sparse_attn_dedup(q, k, v, idx, q_pos0: int, scale: float, out, lse=None, stream=None) -> None:
    """dsa_sparse_attn computed per block of adjacent rows over the union of their index sets."""
    import torch
    bf = torch.bfloat16
    _need(q, bf, "q", (None, None, None))
    Lq, Hq, D = q.shape
    _need(k, bf, "k", (None, None, D))
    _need(v, bf, "v", tuple(k.shape)), _need(idx, torch.int32, "idx", (Lq, None)), _need(out, bf, "out", (Lq, Hq, D))
    if lse is not None:
        _need(lse, torch.float32, "lse", (Lq, Hq))
    _on_device(q=q, k=k, v=v, idx=idx, out=out, lse=lse)
    st = _lib.dsa_sparse_attn_dedup(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), Lq, k.shape[0], q_pos0, Hq, k.shape[1], D,
                                    idx.shape[1], float(scale), _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "dsa_sparse_attn_dedup")


def _prefill_operands(q, k, v, qI, kI, w, out, idx, topk, key_rows, names):
    """Shapes shared by the prefill entry points: q/qI/w/out/idx hold the same query rows, k/v/kI
    at least `key_rows` key rows."""
    import torch
    bf = torch.bfloat16
    nq, nk, nv, nqI, nkI, nw, nout, nidx = names
    _need(q, bf, nq, (None, None, None))
    rows, Hq, D = q.shape
    _need(k, bf, nk, (None, None, D))
    _at_least(k, nk, 0, key_rows)
    _need(v, bf, nv, tuple(k.shape)), _need(qI, bf, nqI, (rows, None, None))
    HI, dI = qI.shape[1], qI.shape[2]
    _need(kI, bf, nkI, (None, dI))
    _at_least(kI, nkI, 0, key_rows)
    _need(w, bf, nw, (rows, HI)), _need(out, bf, nout, (rows, Hq, D))
    if idx is not None:
        _need(idx, torch.int32, nidx, (rows, topk))
    return Hq, D, HI, dI


def dsa_prefill(q, k, v, qI, kI, w, topk: int, scale: float, out, idx_out=None, ws=None, window: int = 0,
                stream=None) -> None:
    """Indexer, top-k and sparse attention for every row of one causal sequence of q.shape[0] tokens."""
    L = q.shape[0] if hasattr(q, "shape") else 0
    Hq, D, HI, dI = _prefill_operands(q, k, v, qI, kI, w, out, idx_out, topk, L,
                                      ("q", "k", "v", "qI", "kI", "w", "out", "idx_out"))
    _on_device(q=q, k=k, v=v, qI=qI, kI=kI, w=w, out=out, idx_out=idx_out, ws=ws)
    ws = _workspace(ws, DSA_OP_PREFILL, L, 1, Hq, HI, topk, q)
    if window:
        st = _lib.dsa_prefill_window(_ptr(q), _ptr(k), _ptr(v), _ptr(qI), _ptr(kI), _ptr(w), L, Hq, k.shape[1], D,
                                     HI, dI, topk, window, float(scale), _ptr(out), _ptr(idx_out), _ptr(ws),
                                     _nbytes(ws), _stream(stream))
        _check(st, "dsa_prefill_window")
        return
    st = _lib.dsa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(qI), _ptr(kI), _ptr(w), L, Hq, k.shape[1], D, HI, dI,
                          topk, float(scale), _ptr(out), _ptr(idx_out), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(st, "dsa_prefill")


def dsa_prefill_rows(q_rows, k, v, qI_rows, kI, w_rows, row0: int, topk: int, scale: float, out_rows,
                     idx_rows=None, ws=None, window: int = 0, stream=None) -> None:
    """Prefill of query rows row0 .. row0+len(q_rows)-1; k, v, kI cover at least those rows."""
    rows = q_rows.shape[0] if hasattr(q_rows, "shape") else 0
    Hq, D, HI, dI = _prefill_operands(q_rows, k, v, qI_rows, kI, w_rows, out_rows, idx_rows, topk, row0 + rows,
                                      ("q_rows", "k", "v", "qI_rows", "kI", "w_rows", "out_rows", "idx_rows"))
    _on_device(q_rows=q_rows, k=k, v=v, qI_rows=qI_rows, kI=kI, w_rows=w_rows, out_rows=out_rows, idx_rows=idx_rows,
               ws=ws)
    ws = _workspace(ws, DSA_OP_PREFILL, row0 + rows, 1, Hq, HI, topk, q_rows)
    st = _lib.dsa_prefill_rows(_ptr(q_rows), _ptr(k), _ptr(v), _ptr(qI_rows), _ptr(kI), _ptr(w_rows), row0, rows, Hq,
                               k.shape[1], D, HI, dI, topk, window, float(scale), _ptr(out_rows), _ptr(idx_rows),
                               _ptr(ws), _nbytes(ws), _stream(stream))
    _check(st, "dsa_prefill_rows")


def dsa_indexer_kl(q, k, qI, kI, w, scale: float, kl, ws=None, stream=None) -> None:
    """Indexer warm-up target KL(P_t || Q_t) for every query row of one causal sequence into kl
    (float32 [L]); see dsa_indexer_kl in include/dsa.h."""
    import torch
    bf = torch.bfloat16
    _need(q, bf, "q", (None, None, None))
    L, Hq, D = q.shape
    _need(k, bf, "k", (None, None, D)), _at_least(k, "k", 0, L), _need(qI, bf, "qI", (L, None, None))
    HI, dI = qI.shape[1], qI.shape[2]
    _need(kI, bf, "kI", (None, dI)), _at_least(kI, "kI", 0, L), _need(w, bf, "w", (L, HI))
    _need(kl, torch.float32, "kl", (None,)), _at_least(kl, "kl", 0, L)
    _on_device(q=q, k=k, qI=qI, kI=kI, w=w, kl=kl, ws=ws)
    ws = _workspace(ws, DSA_OP_INDEXER_KL, L, 1, Hq, HI, 1, q)
    st = _lib.dsa_indexer_kl(_ptr(q), _ptr(k), _ptr(qI), _ptr(kI), _ptr(w), L, Hq, k.shape[1], D, HI, dI,
                             float(scale), _ptr(kl), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(st, "dsa_indexer_kl")


def dsa_decode(q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, topk: int, scale: float, out,
               idx_out=None, ws=None, update_ctx: bool = False, stream=None) -> None:
    """One decode step for B sequences: append the new token at ctx_len[b], then indexer, top-k
    and sparse attention over positions 0 .. ctx_len[b]."""
    import torch
    bf = torch.bfloat16
    _need(q, bf, "q", (None, None, None))
    B, Hq, D = q.shape
    _need(k_cache, bf, "k_cache", (B, None, None, D))
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    _need(v_cache, bf, "v_cache", (B, Lmax, Hkv, D)), _need(qI, bf, "qI", (B, None, None))
    HI, dI = qI.shape[1], qI.shape[2]
    _need(w, bf, "w", (B, HI)), _need(kI_cache, bf, "kI_cache", (B, Lmax, dI))
    _need(k_new, bf, "k_new", (B, Hkv, D)), _need(v_new, bf, "v_new", (B, Hkv, D)), _need(kI_new, bf, "kI_new", (B, dI))
    _need(ctx_len, torch.int32, "ctx_len", (B,)), _need(out, bf, "out", (B, Hq, D))
    if idx_out is not None:
        _need(idx_out, torch.int32, "idx_out", (B, topk))
    _on_device(q=q, qI=qI, w=w, k_new=k_new, v_new=v_new, kI_new=kI_new, k_cache=k_cache, v_cache=v_cache,
               kI_cache=kI_cache, ctx_len=ctx_len, out=out, idx_out=idx_out, ws=ws)
    ws = _workspace(ws, DSA_OP_DECODE, Lmax, B, Hq, HI, topk, q)
    st = _lib.dsa_decode(_ptr(q), _ptr(qI), _ptr(w), _ptr(k_new), _ptr(v_new), _ptr(kI_new), _ptr(k_cache),
                         _ptr(v_cache), _ptr(kI_cache), _ptr(ctx_len), B, Lmax, Hq, Hkv, D, HI, dI, topk,
                         float(scale), int(bool(update_ctx)), _ptr(out), _ptr(idx_out), _ptr(ws), _nbytes(ws),
                         _stream(stream))
    _check(st, "dsa_decode")


def sync_status(stream=None) -> int:
    return int(_lib.dsa_sync_status(_stream(stream)))


def error_site() -> int:
    """Site code (and loop index) of the last device error recorded; 0 if none."""
    return int(_lib.dsa_error_site())


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
