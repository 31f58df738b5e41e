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
    # prefill at 128K: 8192 score rows of 131072 fp32 (4 GiB) + 8192 index rows of 2048 int32
    assert dsa.workspace_size(dsa.DSA_OP_PREFILL, 131072, 1, 32, 32, 2048) == 8192 * 131072 * 4 + 8192 * 2048 * 4
    # small problems: one chunk covering the whole sequence
    assert dsa.workspace_size(dsa.DSA_OP_PREFILL, 1000, 1, 8, 4, 256) == 1000 * 1000 * 4 + 1024000
    assert dsa.workspace_size(dsa.DSA_OP_DECODE, 131328, 16, 32, 32, 2048) >= 16 * 131328 * 4
    assert dsa.workspace_size(dsa.DSA_OP_INDEX, 100) == 0
    # indexer KL at 32K: all 32768 score rows fit in 4 GiB
    assert dsa.workspace_size(dsa.DSA_OP_INDEXER_KL, 32768, 1, 32, 32, 1) == 32768 * 32768 * 4
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
    assert lib.dsa_indexer_kl(*kargs, 64, 4, 128, 32, 64, f, A, A, 1 << 30, None) == dsa.DSA_ERR_UNSUPPORTED
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
