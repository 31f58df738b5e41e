"""Parity at the full workload sizes, in the launch configuration bench.py times (default
workspace: 8192-row chunks at 128K, 4096-row chunks at 256K; decode with 16 sequences, 256 steps
and ctx_len advanced on the device), on sampled rows the oracle computes one by one, plus
properties that hold at any size (index-set structure on every row).

Sampled prefill rows: 1024 drawn uniformly from the sequence plus the boundary rows (first rows,
rows around k, frame/text edges, chunk edges, last rows).  Decode: steps 0, 1, 127 and 255 of
every sequence.  Each checked row must match the oracle's index set outside the near-tie band;
its output must match the oracle evaluated on the GPU's own index set, and, when the two index
sets are equal, the oracle's own output as well."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_output_ok, bf16_tensor_to_f64, index_set_mismatch

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("dsa_lightning_indexer_02_b200")

N_SAMPLED_ROWS = 1024
ORACLE_BATCH = 128            # rows per oracle call (bounds the fp64 score rows kept in memory)
DECODE_CHECK_STEPS = (0, 1, 127, 255)


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


def check_rows_against_oracle(x, rows, gi, go, cfg, what):
    """Rows `rows` of one sequence: GPU indices gi [n, k] and outputs go [n, Hq, D] (float64)
    against the oracle, ORACLE_BATCH rows per call.  Returns summary counts."""
    tot = {"rows": 0, "rows_diff": 0, "keys_diff": 0, "out_of_band": 0, "structural": 0, "same_set_rows": 0}
    worst = {"own_max": 0.0, "ref_max": 0.0}
    for b0 in range(0, len(rows), ORACLE_BATCH):
        r = rows[b0:b0 + ORACLE_BATCH]
        g_idx, g_out = gi[b0:b0 + ORACLE_BATCH], go[b0:b0 + ORACLE_BATCH]
        ref = oracle.dsa_rows(x["q"][r], x["qI"][r], x["w"][r], x["k"], x["v"], x["kI"], r, cfg.k, cfg.scale,
                              keep_scores=True)
        mm = index_set_mismatch(g_idx, ref["idx"], ref["scores"], ref["tau"], ref["absmax"], r + 1)
        assert mm["structural"] == 0 and mm["out_of_band"] == 0, (what, mm)
        for key in ("rows_diff", "keys_diff", "out_of_band", "structural"):
            tot[key] += mm[key]
        tot["rows"] += len(r)
        # headline: the oracle on the GPU's own index sets
        own, _ = oracle.sparse_attn_rows(x["q"][r], x["k"], x["v"], g_idx, cfg.scale)
        e = assert_output_ok(g_out, own, f"{what} (oracle on the GPU's indices)")
        worst["own_max"] = max(worst["own_max"], e["max_abs"])
        # end to end: rows whose set equals the oracle's must also match the oracle's own output
        same = np.array([set(g_idx[i][g_idx[i] >= 0]) == set(ref["idx"][i][ref["idx"][i] >= 0])
                         for i in range(len(r))])
        tot["same_set_rows"] += int(same.sum())
        if same.any():
            e2 = assert_output_ok(g_out[same], ref["out"][same], f"{what} (oracle end to end)")
            worst["ref_max"] = max(worst["ref_max"], e2["max_abs"])
    return tot, worst


def check_full_prefill(name):
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
    del d, srt, valid
    # 1024 uniform rows plus the boundary rows against the oracle
    rows = np.unique(np.concatenate([boundary_rows(cfg), synth.sample_rows(N_SAMPLED_ROWS, L, seed=3)]))
    assert len(rows) >= N_SAMPLED_ROWS
    sel = torch.from_numpy(rows).cuda()
    gi = idx[sel].cpu().numpy()
    go = bf16_tensor_to_f64(out[sel])
    tot, worst = check_rows_against_oracle(x, rows, gi, go, cfg, name)
    print(name, tot, worst)


def test_prefill_128k_sampled(cuda_ok):
    check_full_prefill("128k")


def test_prefill_256k_sampled(cuda_ok):
    check_full_prefill("256k")


def test_decode_16x128k_all_steps(cuda_ok):
    """The bench's decode workload: 16 sequences, 131072 cached tokens each, 256 steps with the
    context length advanced on the device.  Steps 0, 1, 127 and 255 are checked for every
    sequence after the whole loop has run."""
    cfg = synth.CONFIGS["decode"]
    B, ctx0, steps = cfg.batch, cfg.L, cfg.steps
    Lmax = ctx0 + steps
    kc = torch.empty((B, Lmax, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    kIc = torch.empty((B, Lmax, cfg.dI), dtype=torch.bfloat16, device="cuda")
    names = ("q", "qI", "w", "k", "v", "kI")
    new = {n: [] for n in names}
    for b in range(B):
        for n, dst in (("k", kc), ("v", vc), ("kI", kIc)):
            dst[b, :ctx0].copy_(synth.to_torch(synth.tensor(cfg, n, 0, ctx0, seq=b)))
        for n in names:
            new[n].append(synth.to_torch(synth.tensor(cfg, n, ctx0, steps, seq=b)))
    new = {n: torch.stack(new[n], dim=1).cuda().contiguous() for n in names}   # [steps, B, ...]
    ctx = torch.full((B,), ctx0, dtype=torch.int32, device="cuda")
    out = torch.empty((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.workspace_size(dsa.DSA_OP_DECODE, Lmax, B, cfg.Hq, cfg.HI, cfg.k), dtype=torch.uint8,
                     device="cuda")
    kept = {}
    for j in range(steps):
        dsa.dsa_decode(new["q"][j], new["qI"][j], new["w"][j], new["k"][j], new["v"][j], new["kI"][j], kc, vc, kIc,
                       ctx, cfg.k, cfg.scale, out, idx, ws=ws, update_ctx=True)
        if j in DECODE_CHECK_STEPS:
            kept[j] = (idx.cpu().numpy(), bf16_tensor_to_f64(out))
    assert dsa.sync_status() == dsa.DSA_OK
    assert torch.equal(ctx.cpu(), torch.full((B,), ctx0 + steps, dtype=torch.int32))
    del kc, vc, kIc, new
    t_rows = np.array([ctx0 + j for j in DECODE_CHECK_STEPS])
    for b in range(B):
        xb = synth.inputs(cfg, 0, ctx0 + steps, seq=b, names=("k", "v", "kI"))
        for n in ("q", "qI", "w"):               # only the checked tokens' rows
            xb[n] = np.concatenate([synth.tensor(cfg, n, int(t), 1, seq=b) for t in t_rows])
        gi = np.stack([kept[j][0][b] for j in DECODE_CHECK_STEPS])
        go = np.stack([kept[j][1][b] for j in DECODE_CHECK_STEPS])
        ref = oracle.dsa_rows(xb["q"], xb["qI"], xb["w"], xb["k"], xb["v"], xb["kI"], t_rows, cfg.k, cfg.scale,
                              keep_scores=True)
        mm = index_set_mismatch(gi, ref["idx"], ref["scores"], ref["tau"], ref["absmax"], t_rows + 1)
        assert mm["structural"] == 0 and mm["out_of_band"] == 0, (b, mm)
        own, _ = oracle.sparse_attn_rows(xb["q"], xb["k"], xb["v"], gi, cfg.scale)
        assert_output_ok(go, own, f"decode seq {b} (oracle on the GPU's indices)")
        same = np.array([set(gi[i][gi[i] >= 0]) == set(ref["idx"][i][ref["idx"][i] >= 0]) for i in range(len(t_rows))])
        if same.any():
            assert_output_ok(go[same], ref["out"][same], f"decode seq {b} (oracle end to end)")
