"""The C-ABI library loads on a machine without a GPU, exports every symbol the header declares,
and rejects bad arguments on the host before touching CUDA."""
import ctypes

import pytest

import dsa_lightning_indexer_02_b200 as dsa

lib = dsa.lib()


def test_every_header_symbol_is_exported():
    names = dsa.header_symbols()
    assert "dsa_prefill" in names and "dsa_decode" in names and len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    assert dsa.status_string(0) == "DSA_OK"
    for s in range(1, 7):
        assert dsa.status_string(s).startswith("DSA_ERR_")
    assert dsa.status_string(99) == "DSA_ERR_UNKNOWN"
    assert dsa.version() >= 10000


def test_workspace_sizes():
    # prefill at 128K: 32768 score rows of 131072 fp32 (16 GiB) + 32768 index rows of 2048 int32
    assert dsa.workspace_size(dsa.DSA_OP_PREFILL, 131072, 1, 32, 32, 2048) == 32768 * 131072 * 4 + 32768 * 2048 * 4
    # at 256K: 16384 score rows of 262144
    assert dsa.workspace_size(dsa.DSA_OP_PREFILL, 262144, 1, 32, 32, 2048) == 16384 * 262144 * 4 + 16384 * 2048 * 4
    # small problems: one chunk covering the whole sequence
    assert dsa.workspace_size(dsa.DSA_OP_PREFILL, 1000, 1, 8, 4, 256) == 1000 * 1000 * 4 + 1024000
    assert dsa.workspace_size(dsa.DSA_OP_DECODE, 131328, 16, 32, 32, 2048) >= 16 * 131328 * 4
    assert dsa.workspace_size(dsa.DSA_OP_INDEX, 100) == 0
    # indexer KL at 32K: all 32768 score rows fit in 4 GiB
    # (plus each row's 32 per-head log-sum-exps)
    assert dsa.workspace_size(dsa.DSA_OP_INDEXER_KL, 32768, 1, 32, 32, 1) == 32768 * 32768 * 4 + 32768 * 32 * 4
    assert dsa.workspace_size(dsa.DSA_OP_PREFILL, 0) == 0
    assert dsa.workspace_size(99, 100) == 0


P = ctypes.c_void_p


def fake(addr):
    return P(addr)


def test_host_validation_without_gpu():
    A = fake(0x10000)          # 16-byte aligned, never dereferenced: validation fails first
    M = fake(0x10004)          # misaligned
    # null / misaligned pointers
    assert lib.dsa_index(None, A, A, 8, 8, 32, 64, 0, A, 8, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_index(M, A, A, 8, 8, 32, 64, 0, A, 8, None) == dsa.DSA_ERR_INVALID_ARG
    # bad sizes: Lq <= 0, causal rows beyond Lk, ld too small / not a multiple of 4
    assert lib.dsa_index(A, A, A, 0, 8, 32, 64, 0, A, 8, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_index(A, A, A, 8, 4, 32, 64, 0, A, 8, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_index(A, A, A, 8, 8, 32, 64, 0, A, 6, None) == dsa.DSA_ERR_INVALID_ARG
    # unsupported shapes: dI != 64, HI not a power of two <= 64
    assert lib.dsa_index(A, A, A, 8, 8, 32, 128, 0, A, 8, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_index(A, A, A, 8, 8, 24, 64, 0, A, 8, None) == dsa.DSA_ERR_UNSUPPORTED
    # top-k: k = 0 invalid, k too large unsupported
    assert lib.dsa_topk(A, 8, 8, 0, 0, A, None, 0, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk(A, 8, 8, 0, 1 << 20, A, None, 0, None) == dsa.DSA_ERR_UNSUPPORTED
    # attention: D != 128, Hkv = 8, G > 16, Hq % Hkv
    f = ctypes.c_float(0.1)
    assert lib.dsa_sparse_attn(A, A, A, A, 4, 4, 0, 32, 4, 64, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn(A, A, A, A, 4, 4, 0, 64, 8, 128, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn(A, A, A, A, 4, 4, 0, 34, 2, 128, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn(A, A, A, A, 4, 4, 0, 30, 4, 128, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn(A, A, A, A, 4, 4, 0, 32, 4, 128, 0, f, A, None, None) == dsa.DSA_ERR_INVALID_ARG
    nan = ctypes.c_float(float("nan"))
    assert lib.dsa_sparse_attn(A, A, A, A, 4, 4, 0, 32, 4, 128, 16, nan, A, None, None) == dsa.DSA_ERR_INVALID_ARG
    # dedup attention: the per-token checks, and G = Hq / Hkv must be 8 or 16
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 4, 4, 0, 32, 4, 64, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 4, 4, 0, 16, 4, 128, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 4, 4, 0, 8, 4, 128, 16, f, A, None, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 0, 4, 0, 32, 4, 128, 16, f, A, None, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 4, 4, 0, 32, 4, 128, 0, f, A, None, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_attn_dedup(None, A, A, A, 4, 4, 0, 32, 4, 128, 16, f, A, None, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 4, 4, 0, 32, 4, 128, 16, nan, A, None, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_attn_dedup(A, A, A, A, 4, (1 << 31) - 100, 0, 32, 4, 128, 16, f, A, None, None) == \
        dsa.DSA_ERR_UNSUPPORTED
    # prefill: workspace missing / too small
    args = [A] * 6 + [1024, 32, 4, 128, 32, 64, 2048, f, A, None]
    assert lib.dsa_prefill(*args, None, 0, None) == dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_prefill(*args, A, 64, None) == dsa.DSA_ERR_WORKSPACE
    # decode: HI must be 16/32/64; workspace must fit
    dargs = [A] * 10
    assert lib.dsa_decode(*dargs, 4, 4096, 32, 4, 128, 4, 64, 2048, f, 0, A, None, A, 1 << 30, None) == \
        dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_decode(*dargs, 4, 4096, 32, 4, 128, 32, 64, 2048, f, 0, A, None, A, 1024, None) == \
        dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_decode(*dargs, 0, 4096, 32, 4, 128, 32, 64, 2048, f, 0, A, None, A, 1 << 30, None) == \
        dsa.DSA_ERR_INVALID_ARG
    # indexer KL: pointers, shapes, workspace
    kargs = [A] * 5 + [1024]
    assert lib.dsa_indexer_kl(None, *[A] * 4, 1024, 32, 4, 128, 32, 64, f, A, A, 1 << 30, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_indexer_kl(*kargs, 32, 4, 64, 32, 64, f, A, A, 1 << 30, None) == dsa.DSA_ERR_UNSUPPORTED
    # KL: Hq must be 8/16/32/64 with at least two query heads per KV group
    assert lib.dsa_indexer_kl(*kargs, 4, 4, 128, 32, 64, f, A, A, 1 << 30, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_indexer_kl(*kargs, 24, 4, 128, 32, 64, f, A, A, 1 << 30, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_indexer_kl(*kargs, 8, 8, 128, 32, 64, f, A, A, 1 << 30, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_indexer_kl(*kargs, 32, 4, 128, 32, 64, f, A, None, 0, None) == dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_indexer_kl(*kargs, 32, 4, 128, 32, 64, f, A, A, 64, None) == dsa.DSA_ERR_WORKSPACE
    # self test bounds
    assert lib.dsa_selftest_timeout(0, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_selftest_timeout(3_000_000_000, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_launch_count() == 0


def test_torch_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 32, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dsa.dsa_index(x, torch.zeros(4, 64, dtype=torch.bfloat16), torch.zeros(4, 32, dtype=torch.bfloat16), 0,
                      torch.zeros(4, 4))


def _bf(*shape):
    import torch
    return torch.zeros(shape, dtype=torch.bfloat16)


def _i32(*shape):
    import torch
    return torch.zeros(shape, dtype=torch.int32)


def _f32(*shape):
    import torch
    return torch.zeros(shape, dtype=torch.float32)


def _prefill_args(L=16, Hq=8, Hkv=2, D=128, HI=4, dI=64, k=8):
    return dict(q=_bf(L, Hq, D), k=_bf(L, Hkv, D), v=_bf(L, Hkv, D), qI=_bf(L, HI, dI), kI=_bf(L, dI),
                w=_bf(L, HI), topk=k, scale=0.1, out=_bf(L, Hq, D), idx_out=_i32(L, k))


def _decode_args(B=2, Lmax=32, Hq=8, Hkv=2, D=128, HI=16, dI=64, k=8):
    return dict(q=_bf(B, Hq, D), qI=_bf(B, HI, dI), w=_bf(B, HI), k_new=_bf(B, Hkv, D), v_new=_bf(B, Hkv, D),
                kI_new=_bf(B, dI), k_cache=_bf(B, Lmax, Hkv, D), v_cache=_bf(B, Lmax, Hkv, D),
                kI_cache=_bf(B, Lmax, dI), ctx_len=_i32(B), topk=k, scale=0.1, out=_bf(B, Hq, D),
                idx_out=_i32(B, k))


# (entry point, consistent arguments, {operand: a wrong-shaped replacement})
_SHAPE_CASES = [
    (dsa.dsa_index, dict(qI=_bf(8, 4, 64), kI=_bf(8, 64), w=_bf(8, 4), q_pos0=0, scores=_f32(8, 8)),
     {"kI": _bf(8, 32), "w": _bf(8, 5), "scores": _f32(7, 8)}),
    (dsa.dsa_topk, dict(scores=_f32(8, 8), q_pos0=0, k=4, idx=_i32(8, 4)),
     {"idx": _i32(8, 5)}),
    (dsa.dsa_sparse_attn, dict(q=_bf(8, 8, 128), k=_bf(8, 2, 128), v=_bf(8, 2, 128), idx=_i32(8, 4), q_pos0=0,
                               scale=0.1, out=_bf(8, 8, 128), lse=_f32(8, 8)),
     {"k": _bf(8, 2, 64), "v": _bf(9, 2, 128), "idx": _i32(7, 4), "out": _bf(8, 4, 128), "lse": _f32(8, 4)}),
    (dsa.dsa_sparse_attn_dedup, dict(q=_bf(8, 16, 128), k=_bf(8, 2, 128), v=_bf(8, 2, 128), idx=_i32(8, 4),
                                     q_pos0=0, scale=0.1, out=_bf(8, 16, 128), lse=_f32(8, 16)),
     {"k": _bf(8, 2, 64), "v": _bf(9, 2, 128), "idx": _i32(7, 4), "out": _bf(8, 8, 128), "lse": _f32(8, 8)}),
    (dsa.dsa_prefill, _prefill_args(),
     {"k": _bf(15, 2, 128), "v": _bf(16, 1, 128), "qI": _bf(15, 4, 64), "kI": _bf(16, 32), "w": _bf(16, 3),
      "out": _bf(16, 8, 64), "idx_out": _i32(16, 9)}),
    (dsa.dsa_indexer_kl, dict(q=_bf(16, 8, 128), k=_bf(16, 2, 128), qI=_bf(16, 4, 64), kI=_bf(16, 64),
                              w=_bf(16, 4), scale=0.1, kl=_f32(16)),
     {"k": _bf(15, 2, 128), "qI": _bf(15, 4, 64), "kI": _bf(15, 64), "w": _bf(16, 8), "kl": _f32(15)}),
    (dsa.dsa_decode, _decode_args(),
     {"qI": _bf(3, 16, 64), "w": _bf(2, 8), "k_new": _bf(2, 1, 128), "v_new": _bf(2, 2, 64), "kI_new": _bf(2, 32),
      "k_cache": _bf(2, 32, 2, 64), "v_cache": _bf(2, 31, 2, 128), "kI_cache": _bf(2, 32, 32), "ctx_len": _i32(3),
      "out": _bf(2, 8, 64), "idx_out": _i32(2, 7)}),
]


@pytest.mark.parametrize("fn,args,bad", _SHAPE_CASES, ids=[c[0].__name__ for c in _SHAPE_CASES])
def test_binding_checks_every_operand_shape(fn, args, bad):
    """A consistent call gets past the shape checks (and stops at the CPU-tensor check); each
    operand whose shape disagrees with the leading one is refused by name before any pointer is
    passed on."""
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn(**args)
    for name, wrong in bad.items():
        with pytest.raises(ValueError, match=f"^{name}"):
            fn(**{**args, name: wrong})


def test_binding_prefill_rows_needs_keys_up_to_its_last_row():
    a = _prefill_args()
    rows = dict(q_rows=a["q"][:8], k=a["k"], v=a["v"], qI_rows=a["qI"][:8], kI=a["kI"], w_rows=a["w"][:8],
                topk=8, scale=0.1, out_rows=a["out"][:8], idx_rows=a["idx_out"][:8])
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        dsa.dsa_prefill_rows(row0=8, **rows)
    with pytest.raises(ValueError, match=r"^k\.shape\[0\] must be >= 17"):
        dsa.dsa_prefill_rows(row0=9, **rows)


def _c_kind(decl: str) -> str:
    """Coarse ctypes kind of one C parameter or return type from include/dsa.h."""
    d = " ".join(decl.replace("const", " ").split())
    if "*" in d or d.startswith("dsa_stream_t"):
        return "ptr"
    base = d.split()[0]
    if d.startswith("unsigned int"):
        return "uint"
    return {"int": "int", "int64_t": "i64", "size_t": "size", "float": "float", "double": "double",
            "dsa_status": "int", "void": "void"}[base]


_CTYPES_KIND = {ctypes.c_void_p: "ptr", ctypes.c_char_p: "ptr", ctypes.c_int: "int", ctypes.c_uint: "uint",
                ctypes.c_int64: "i64",
                ctypes.c_size_t: "size", ctypes.c_float: "float", ctypes.c_double: "double", None: "void"}


def test_binding_signatures_match_the_header():
    """Every prototype in include/dsa.h and the binding's ctypes signature of the same name agree
    in return kind, argument count and each argument's kind (a pointer passed where the header
    expects a size, or a dropped argument, would reach a kernel as a bad address)."""
    import re
    with open(dsa.HEADER_PATH) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    decls = re.findall(r"([A-Za-z_][\w \*]*?)\b(dsa_[a-z_]+)\s*\(([^)]*)\)\s*;", text)
    assert len(decls) == len(dsa.header_symbols())
    for ret, name, params in decls:
        params = params.strip()
        kinds = [] if params in ("", "void") else [_c_kind(p) for p in params.split(",")]
        res, args = dsa._SIGS[name]
        assert _CTYPES_KIND[res] == _c_kind(ret.strip()), name
        assert [_CTYPES_KIND[a] for a in args] == kinds, name


def test_host_validation_of_window_rows_and_noalloc_entry_points():
    """The variants of prefill, top-k and decode refuse bad sizes, windows and workspaces on the
    host, before any CUDA call."""
    A = fake(0x10000)
    f = 0.1
    # top-k with a window: negative window, k = 0, rows past ld
    assert lib.dsa_topk_window(A, 8, 8, 0, 4, -1, A, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_window(A, 8, 8, 0, 0, 16, A, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_window(A, 8, 8, 4, 4, 16, A, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_window(A, 8, 8, 0, 1 << 20, 16, A, None) == dsa.DSA_ERR_UNSUPPORTED
    # prefill of a row range: empty range, negative row0 or window, missing workspace
    shape = [32, 4, 128, 32, 64, 2048]                     # Hq, Hkv, D, HI, dI, topk
    def rows(row0, n, window, ws=A, ws_bytes=1 << 40):
        return lib.dsa_prefill_rows(*[A] * 6, row0, n, *shape, window, f, A, None, ws, ws_bytes, None)
    assert rows(0, 0, 0) == dsa.DSA_ERR_INVALID_ARG
    assert rows(-1, 8, 0) == dsa.DSA_ERR_INVALID_ARG
    assert rows(0, 8, -5) == dsa.DSA_ERR_INVALID_ARG
    assert rows(0, 8, 0, ws=None, ws_bytes=0) == dsa.DSA_ERR_WORKSPACE
    assert rows(0, 4096, 0, ws_bytes=1024) == dsa.DSA_ERR_WORKSPACE
    # windowed prefill: empty sequence, and the shape checks it shares with prefill
    assert lib.dsa_prefill_window(*[A] * 6, 0, *shape, 100, f, A, None, A, 1 << 30, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_prefill_window(*[A] * 6, 1024, 32, 4, 64, 32, 64, 2048, 100, f, A, None, A, 1 << 30, None) == \
        dsa.DSA_ERR_UNSUPPORTED
    # allocation-free decode: bad batch, and a step too large for its fixed scratch
    dargs = [A] * 10
    assert lib.dsa_decode_noalloc(*dargs, 0, 4096, 32, 4, 128, 32, 64, 2048, f, 0, A, None, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_decode_noalloc(*dargs, 256, 1 << 22, 32, 4, 128, 32, 64, 2048, f, 0, A, None, None) == \
        dsa.DSA_ERR_WORKSPACE
    # argument errors before the scratch-size check, with dsa_decode's codes
    assert lib.dsa_decode_noalloc(*dargs, 256, 1 << 22, 32, 4, 128, 32, 64, 1 << 20, f, 0, A, None, None) == \
        dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_decode_noalloc(*dargs, 256, 1 << 22, 32, 4, 128, 24, 64, 2048, f, 0, A, None, None) == \
        dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_decode_noalloc(None, *dargs[1:], 256, 1 << 22, 32, 4, 128, 32, 64, 2048, f, 0, A, None, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_decode_noalloc(*dargs, 256, 1 << 22, 32, 4, 128, 32, 64, 2048, f, 0, fake(0x10008), None, None) == \
        dsa.DSA_ERR_INVALID_ARG
    # the decode workload (16 sequences of 131072 + 256 positions) fits the fixed array even with
    # the index rows kept in it
    assert dsa.workspace_size(dsa.DSA_OP_DECODE, 131072 + 256, 16, 32, 32, 2048) <= \
        int(lib.dsa_decode_noalloc_scratch_bytes())
    assert lib.dsa_launch_count() == 0
