"""dsa_decode_noalloc: the decode step for callers that cannot allocate device memory.

Some callers have no way to obtain a workspace -- a plugin inside a serving process whose
memory pool owns the GPU, or a latency-critical path that must not pay cudaMalloc's implicit
device synchronisation.  dsa_decode_noalloc runs the same decode step as dsa_decode with its
scratch in a fixed array inside the library.  This test calls it through the C ABI and checks,
on two decode steps in a row, that it gives what dsa_decode gives on an identical copy of the
state (same index sets, outputs within the tolerances of the other parity tests), both when the
caller passes idx_out and when the index rows stay in the fixed array, and that a problem too
large for the fixed array is refused without a launch (argument errors first, as dsa_decode).

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from parity import assert_output_ok, bf16_tensor_to_f64

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("dsa_lightning_indexer_02_b200")


def ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def call_noalloc(new, kc, vc, kIc, ctx, cfg, out, idx, update_ctx=1):
    B, Lmax = kc.shape[0], kc.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return dsa.lib().dsa_decode_noalloc(ptr(new["q"]), ptr(new["qI"]), ptr(new["w"]), ptr(new["k"]), ptr(new["v"]),
                                        ptr(new["kI"]), ptr(kc), ptr(vc), ptr(kIc), ptr(ctx), B, Lmax, cfg.Hq,
                                        cfg.Hkv, cfg.D, cfg.HI, cfg.dI, cfg.k, ctypes.c_float(cfg.scale),
                                        update_ctx, ptr(out), ptr(idx), stream)


@pytest.mark.parametrize("own_idx", [True, False], ids=["idx_out", "idx_in_scratch"])
def test_noalloc_decode_matches_dsa_decode_on_two_steps(cuda_ok, own_idx):
    """With idx_out given, and with idx_out NULL (the index rows then live in the fixed array
    between the top-k and the attention kernels): two steps in a row give dsa_decode's results."""
    cfg = synth.CONFIGS["32k"]
    B, Lmax, steps = 4, 6144, 2
    ctx0 = np.array([5, 1500, 2047, 6000])
    data = [synth.inputs(cfg, 0, int(ctx0[b]) + steps, seq=b) for b in range(B)]
    kc = torch.zeros((B, Lmax, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kIc = torch.zeros((B, Lmax, cfg.dI), dtype=torch.bfloat16, device="cuda")
    for b in range(B):
        c = int(ctx0[b])
        kc[b, :c] = synth.to_torch(data[b]["k"][:c]).cuda()
        vc[b, :c] = synth.to_torch(data[b]["v"][:c]).cuda()
        kIc[b, :c] = synth.to_torch(data[b]["kI"][:c]).cuda()
    state_a = [t.clone() for t in (kc, vc, kIc)]          # reference: dsa_decode + caller workspace
    state_b = [t.clone() for t in (kc, vc, kIc)]          # dsa_decode_noalloc
    ctx_a = torch.from_numpy(ctx0.astype(np.int32)).cuda()
    ctx_b = ctx_a.clone()
    ws = torch.empty(dsa.workspace_size(dsa.DSA_OP_DECODE, Lmax, B, cfg.Hq, cfg.HI, cfg.k), dtype=torch.uint8,
                     device="cuda")
    for j in range(steps):
        pos = ctx0 + j
        new = {n: synth.to_torch(np.stack([data[b][n][pos[b]] for b in range(B)])).cuda()
               for n in ("q", "qI", "w", "k", "v", "kI")}
        out_a = torch.empty((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
        idx_a = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
        dsa.dsa_decode(new["q"], new["qI"], new["w"], new["k"], new["v"], new["kI"], *state_a, ctx_a, cfg.k,
                       cfg.scale, out_a, idx_a, ws=ws, update_ctx=True)
        out_b = torch.full_like(out_a, float("nan"))
        idx_b = torch.full_like(idx_a, -7) if own_idx else None
        st = call_noalloc(new, *state_b, ctx_b, cfg, out_b, idx_b)
        assert st == dsa.DSA_OK, dsa.status_string(st)
        assert dsa.sync_status() == dsa.DSA_OK
        assert torch.equal(ctx_a, ctx_b) and np.array_equal(ctx_b.cpu().numpy(), pos + 1)
        if own_idx:
            for b in range(B):
                assert sorted(idx_a[b].tolist()) == sorted(idx_b[b].tolist()), (j, b)
        assert_output_ok(bf16_tensor_to_f64(out_b), bf16_tensor_to_f64(out_a), f"step {j}")
        for a, b_ in zip(state_a, state_b):              # the appended cache rows agree too
            assert torch.equal(a.view(torch.int16), b_.view(torch.int16))


def test_noalloc_decode_refuses_problems_beyond_its_scratch(cuda_ok):
    cfg = synth.CONFIGS["32k"]
    limit = int(dsa.lib().dsa_decode_noalloc_scratch_bytes())
    assert limit == 16 << 20
    B, Lmax = 64, 131072                                    # 64 score rows of 131072 fp32 = 32 MiB
    assert dsa.workspace_size(dsa.DSA_OP_DECODE, Lmax, B, cfg.Hq, cfg.HI, cfg.k) > limit
    one = torch.zeros(16, dtype=torch.bfloat16, device="cuda")   # never read: refused before any launch
    ctx = torch.zeros(B, dtype=torch.int32, device="cuda")
    n0 = dsa.launch_count()
    new = {n: one for n in ("q", "qI", "w", "k", "v", "kI")}
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = dsa.lib().dsa_decode_noalloc(ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one),
                                      ptr(one), ptr(ctx), B, Lmax, cfg.Hq, cfg.Hkv, cfg.D, cfg.HI, cfg.dI, cfg.k,
                                      ctypes.c_float(cfg.scale), 0, ptr(one), None, stream)
    assert st == dsa.DSA_ERR_WORKSPACE
    # argument errors come first, exactly as dsa_decode reports them
    st = dsa.lib().dsa_decode_noalloc(ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one),
                                      ptr(one), ptr(ctx), B, Lmax, cfg.Hq, cfg.Hkv, cfg.D, cfg.HI, cfg.dI, 1 << 20,
                                      ctypes.c_float(cfg.scale), 0, ptr(one), None, stream)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    st = dsa.lib().dsa_decode_noalloc(None, ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one), ptr(one),
                                      ptr(one), ptr(ctx), B, Lmax, cfg.Hq, cfg.Hkv, cfg.D, cfg.HI, cfg.dI, cfg.k,
                                      ctypes.c_float(cfg.scale), 0, ptr(one), None, stream)
    assert st == dsa.DSA_ERR_INVALID_ARG
    assert dsa.launch_count() == n0
    assert dsa.sync_status() == dsa.DSA_OK
