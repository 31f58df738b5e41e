"""Parity at the full workload sizes, in the launch configuration bench.py times (default
workspace: 8192-row chunks at 128K, 4096-row chunks at 256K; decode with 16 sequences and
ctx_len advanced on the device), on sampled rows the oracle computes one by one, plus
properties that hold at any size (index-set structure on every row)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_output_ok, bf16_tensor_to_f64, index_set_mismatch

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("dsa_lightning_indexer_02_b200")


def dev(a):
    return synth.to_torch(a).cuda()


def boundary_rows(cfg):
    L, k = cfg.L, cfg.k
    rows = [0, 1, k - 2, k - 1, k, k + 1, L - 2, L - 1]
    if cfg.layout == synth.LAYOUT_FRAME_TEXT:           # frame/text edges of the 512+64 layout
        rows += [511, 512, 575, 576, 576 * 100 + 511, 576 * 100 + 512]
    elif cfg.layout == synth.LAYOUT_TEXT_FRAME:         # text/frame edges of the 16+240 layout
        rows += [15, 16, 255, 256, 256 * 500 + 15, 256 * 500 + 16]
    chunk = 8192 if L <= 131072 else 4096               # default-workspace chunk edges
    rows += [chunk - 1, chunk, L - chunk - 1, L - chunk]
    return rows


def check_full_prefill(name, n_sample):
    cfg = synth.CONFIGS[name]
    x = synth.inputs(cfg, 0, cfg.L)
    L = cfg.L
    out = torch.empty((L, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
    d = {n: dev(a) for n, a in x.items()}
    dsa.dsa_prefill(d["q"], d["k"], d["v"], d["qI"], d["kI"], d["w"], cfg.k, cfg.scale, out, idx)
    assert dsa.sync_status() == dsa.DSA_OK
    # properties on every row: sets of min(k, t+1) distinct causal keys, -1 padded
    t = torch.arange(L, device="cuda", dtype=torch.int64)
    valid = idx >= 0
    assert torch.equal(valid.sum(1), torch.clamp(t + 1, max=cfg.k))
    assert bool(((idx.long() <= t[:, None]) | ~valid).all())
    srt = torch.sort(idx.long(), dim=1).values
    assert int(((srt[:, 1:] == srt[:, :-1]) & (srt[:, 1:] >= 0)).sum()) == 0
    assert bool(torch.isfinite(out.float()).all())
    # sampled rows against the oracle
    rows = np.unique(np.concatenate([boundary_rows(cfg), synth.sample_rows(n_sample, L, seed=3)]))
    ref = oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows, cfg.k,
                          cfg.scale, keep_scores=True)
    sel = torch.from_numpy(rows).cuda()
    gi = idx[sel].cpu().numpy()
    mm = index_set_mismatch(gi, ref["idx"], ref["scores"], ref["tau"], ref["absmax"], rows + 1)
    assert mm["structural"] == 0 and mm["out_of_band"] == 0, mm
    own, _ = oracle.sparse_attn_rows(x["q"][rows], x["k"], x["v"], gi, cfg.scale)
    e = assert_output_ok(bf16_tensor_to_f64(out[sel]), own, name)
    print(name, len(rows), "rows", mm, e)


def test_prefill_128k_sampled(cuda_ok):
    check_full_prefill("128k", 24)


def test_prefill_256k_sampled(cuda_ok):
    check_full_prefill("256k", 12)


def test_decode_16x128k_sampled(cuda_ok):
    cfg = synth.CONFIGS["decode"]
    B, ctx0, steps = cfg.batch, cfg.L, 3
    Lmax = ctx0 + cfg.steps
    kc = torch.empty((B, Lmax, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    kIc = torch.empty((B, Lmax, cfg.dI), dtype=torch.bfloat16, device="cuda")
    data = []
    for b in range(B):
        xb = synth.inputs(cfg, 0, ctx0 + steps, seq=b)
        data.append(xb)
        kc[b, :ctx0].copy_(synth.to_torch(xb["k"][:ctx0]))
        vc[b, :ctx0].copy_(synth.to_torch(xb["v"][:ctx0]))
        kIc[b, :ctx0].copy_(synth.to_torch(xb["kI"][:ctx0]))
    ctx = torch.full((B,), ctx0, dtype=torch.int32, device="cuda")
    out = torch.empty((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.workspace_size(dsa.DSA_OP_DECODE, Lmax, B, cfg.Hq, cfg.HI, cfg.k), dtype=torch.uint8,
                     device="cuda")
    check = {0: range(B), steps - 1: (0, 5, 10, 15)}
    for j in range(steps):
        t = ctx0 + j
        new = {n: dev(np.stack([data[b][n][t] for b in range(B)])) for n in ("q", "qI", "w", "k", "v", "kI")}
        dsa.dsa_decode(new["q"], new["qI"], new["w"], new["k"], new["v"], new["kI"], kc, vc, kIc, ctx, cfg.k,
                       cfg.scale, out, idx, ws=ws, update_ctx=True)
        assert dsa.sync_status() == dsa.DSA_OK
        if j not in check:
            continue
        gi, go = idx.cpu().numpy(), bf16_tensor_to_f64(out)
        for b in check[j]:
            xb, r = data[b], np.array([t])
            ref = oracle.dsa_rows(xb["q"][r], xb["qI"][r], xb["w"][r], xb["k"], xb["v"], xb["kI"], r, cfg.k,
                                  cfg.scale, keep_scores=True)
            mm = index_set_mismatch(gi[b:b + 1], ref["idx"], ref["scores"], ref["tau"], ref["absmax"], r + 1)
            assert mm["structural"] == 0 and mm["out_of_band"] == 0, (b, j, mm)
            own, _ = oracle.sparse_attn_rows(xb["q"][r], xb["k"], xb["v"], gi[b:b + 1], cfg.scale)
            assert_output_ok(go[b:b + 1], own, f"decode b={b} step={j}")
    assert torch.equal(ctx.cpu(), torch.full((B,), ctx0 + steps, dtype=torch.int32))
