"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle, step by step and fused.

Sizes: the whole 'tiny' workload (L=1024, k=256, 8/2/128, HI=4) and slices / the whole of the
'32k' workload (L=32768, k=2048, 32/4/128, HI=32), so that the kernels run over many tiles plus
ragged tails.  Tolerances: see tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_output_ok, bf16_tensor_to_f64, index_set_mismatch

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("dsa_lightning_indexer_02_b200")


def dev(a: np.ndarray) -> torch.Tensor:
    return synth.to_torch(a).cuda()


def score_bound(qI, w, kI, t_rows):
    """|fp32 score - exact score| bound: 64 u * sum_h |w_h| sum_d |q_hd k_d| (fp32 MMA sum of 64
    exact products) + 32 u * sum_h |w_h| relu_h (fp32 head sum), u = 2^-24; taken as 1e-5 * B."""
    qa = np.abs(synth.bf16_to_f64(qI))          # [r, HI, dI]
    wa = np.abs(synth.bf16_to_f64(w))           # [r, HI]
    ka = np.abs(synth.bf16_to_f64(kI))          # [Lk, dI]
    return np.einsum("rh,rhd,sd->rs", wa, qa, ka[: int(np.max(t_rows)) + 1])


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.CONFIGS["tiny"]
    x = synth.inputs(cfg, 0, cfg.L)
    rows = np.arange(cfg.L)
    ref = oracle.dsa_rows(x["q"], x["qI"], x["w"], x["k"], x["v"], x["kI"], rows, cfg.k, cfg.scale,
                          keep_scores=True)
    return cfg, x, ref


def test_index_tiny_full(cuda_ok, tiny):
    cfg, x, ref = tiny
    L = cfg.L
    scores = torch.full((L, L), float("nan"), device="cuda")
    dsa.dsa_index(dev(x["qI"]), dev(x["kI"]), dev(x["w"]), 0, scores)
    assert dsa.sync_status() == dsa.DSA_OK
    got = scores.cpu().double().numpy()
    mask = np.tril(np.ones((L, L), dtype=bool))
    bound = 1e-5 * score_bound(x["qI"], x["w"], x["kI"], np.arange(L)) + 1e-30
    err = np.abs(got - ref["scores"])
    assert np.all(err[mask] <= bound[mask]), float(np.max(err[mask] / bound[mask]))
    assert np.all(np.isnan(got[~mask]))  # nothing written above the diagonal


@pytest.mark.parametrize("q_pos0,Lq", [(32768 - 96, 96), (1000, 37), (0, 5)])
def test_index_32k_slices(cuda_ok, q_pos0, Lq):
    cfg = synth.CONFIGS["32k"]
    Lk = q_pos0 + Lq
    qI, w = synth.tensor(cfg, "qI", q_pos0, Lq), synth.tensor(cfg, "w", q_pos0, Lq)
    kI = synth.tensor(cfg, "kI", 0, Lk)
    ld = (Lk + 3) // 4 * 4
    scores = torch.full((Lq, ld), float("nan"), device="cuda")
    dsa.dsa_index(dev(qI), dev(kI), dev(w), q_pos0, scores)
    assert dsa.sync_status() == dsa.DSA_OK
    rows = np.arange(q_pos0, q_pos0 + Lq)
    ref = oracle.index_rows(qI, w, kI, rows)
    got = scores.cpu().double().numpy()[:, :Lk]
    bound = 1e-5 * score_bound(qI, w, kI, rows)
    for r in range(Lq):
        n = rows[r] + 1
        assert np.all(np.abs(got[r, :n] - ref[r, :n]) <= bound[r, :n]), r
        assert np.all(np.isnan(got[r, n:]))


def test_topk_exact_on_oracle_scores(cuda_ok, tiny):
    """Fed the oracle's scores rounded to fp32, the GPU top-k must equal the oracle's top-k of the
    same fp32 values exactly (ties by lower index)."""
    cfg, x, ref = tiny
    L = cfg.L
    s32 = np.nan_to_num(ref["scores"], nan=0.0).astype(np.float32)
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(torch.from_numpy(s32).cuda(), 0, cfg.k, idx)
    assert dsa.sync_status() == dsa.DSA_OK
    want, _ = oracle.topk_rows(s32.astype(np.float64), np.arange(L) + 1, cfg.k)
    got = idx.cpu().numpy()
    for r in range(L):
        assert sorted(got[r][got[r] >= 0].tolist()) == sorted(want[r][want[r] >= 0].tolist()), r
        assert np.all(got[r][min(cfg.k, r + 1):] == -1)


@pytest.mark.parametrize("kind", ["ties", "zeros", "wide"])
def test_topk_long_rows_and_heavy_ties(cuda_ok, kind):
    """Long rows (beyond the candidate buffer), massive exact ties, -0/+0, the global-memory path."""
    rng = np.random.default_rng(11)
    rows, n, k = 6, 40000, 2048
    ld = n
    if kind == "ties":
        s = rng.integers(-3, 4, size=(rows, ld)).astype(np.float32)       # 7 distinct values
    elif kind == "zeros":
        s = np.zeros((rows, ld), dtype=np.float32)
        s[:, ::7] = -0.0
        s[:, 5::11] = 1.0
    else:
        s = (rng.standard_normal((rows, ld)) * 30).astype(np.float32)
    q_pos0 = n - rows
    idx = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(torch.from_numpy(s).cuda(), q_pos0, k, idx)
    assert dsa.sync_status() == dsa.DSA_OK
    want, _ = oracle.topk_rows(s.astype(np.float64), q_pos0 + np.arange(rows) + 1, k)
    got = idx.cpu().numpy()
    for r in range(rows):
        assert sorted(got[r].tolist()) == sorted(want[r].tolist()), r


def test_sparse_attn_on_oracle_indices(cuda_ok, tiny):
    cfg, x, ref = tiny
    L = cfg.L
    out = torch.empty((L, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((L, cfg.Hq), dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_attn(dev(x["q"]), dev(x["k"]), dev(x["v"]), torch.from_numpy(ref["idx"]).cuda(), 0, cfg.scale,
                        out, lse)
    assert dsa.sync_status() == dsa.DSA_OK
    assert_output_ok(bf16_tensor_to_f64(out), ref["out"], "attn")
    np.testing.assert_allclose(lse.cpu().numpy(), ref["lse"], rtol=0, atol=2e-3)


def test_sparse_attn_gqa_shapes(cuda_ok):
    """G = 16 (two 8-head tiles), Hkv = 1 and 2, topk not a multiple of the stage size."""
    rng = np.random.default_rng(12)
    for Hq, Hkv, topk in ((32, 2, 300), (16, 1, 77), (8, 4, 129)):
        L = 700
        q = rng.standard_normal((L, Hq, 128)).astype(np.float32)
        k = rng.standard_normal((L, Hkv, 128)).astype(np.float32)
        v = rng.standard_normal((L, Hkv, 128)).astype(np.float32)
        tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16) for a in (q, k, v))
        bits = [t.view(torch.int16).numpy().view(np.uint16) for t in (tq, tk, tv)]
        idx = np.full((L, topk), -1, dtype=np.int32)
        for t in range(L):
            m = min(topk, t + 1)
            idx[t, :m] = rng.choice(t + 1, size=m, replace=False)
        out = torch.empty((L, Hq, 128), dtype=torch.bfloat16, device="cuda")
        dsa.dsa_sparse_attn(tq.cuda(), tk.cuda(), tv.cuda(), torch.from_numpy(idx).cuda(), 0, 0.0883883, out)
        assert dsa.sync_status() == dsa.DSA_OK
        want, _ = oracle.sparse_attn_rows(bits[0], bits[1], bits[2], idx, 0.0883883)
        assert_output_ok(bf16_tensor_to_f64(out), want, f"Hq={Hq} Hkv={Hkv}")


def check_prefill(cfg, x, idx_gpu, out_gpu, rows):
    """Index sets within the near-tie band and outputs within tolerance on sampled rows."""
    ref = oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows, cfg.k,
                          cfg.scale, keep_scores=True)
    mm = index_set_mismatch(idx_gpu, ref["idx"], ref["scores"], ref["tau"], ref["absmax"], rows + 1)
    assert mm["structural"] == 0 and mm["out_of_band"] == 0, mm
    own, _ = oracle.sparse_attn_rows(x["q"][rows], x["k"], x["v"], idx_gpu, cfg.scale)
    assert_output_ok(out_gpu, own, "vs oracle on GPU indices")
    if mm["rows_diff"] == 0:
        assert_output_ok(out_gpu, ref["out"], "vs oracle end to end")
    return mm


def run_prefill(cfg, x, ws_bytes=None):
    L = cfg.L
    out = torch.empty((L, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
    ws = None
    if ws_bytes is not None:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    dsa.dsa_prefill(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["qI"]), dev(x["kI"]), dev(x["w"]), cfg.k,
                    cfg.scale, out, idx, ws)
    assert dsa.sync_status() == dsa.DSA_OK
    return out, idx


def test_prefill_tiny_full(cuda_ok, tiny):
    cfg, x, ref = tiny
    out, idx = run_prefill(cfg, x)
    rows = np.arange(cfg.L)
    check_prefill(cfg, x, idx.cpu().numpy(), bf16_tensor_to_f64(out), rows)


def test_prefill_tiny_chunked_is_identical_and_deterministic(cuda_ok, tiny):
    cfg, x, _ = tiny
    out1, idx1 = run_prefill(cfg, x)
    per_row = cfg.L * 4
    out2, idx2 = run_prefill(cfg, x, ws_bytes=200 * per_row + 4096)   # chunks of 192 rows
    out3, idx3 = run_prefill(cfg, x)
    for a, b in ((out1, out2), (out1, out3)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(idx1, idx2) and torch.equal(idx1, idx3)


@pytest.fixture(scope="module")
def c32k():
    cfg = synth.CONFIGS["32k"]
    return cfg, synth.inputs(cfg, 0, cfg.L)


def test_prefill_32k_sampled_rows(cuda_ok, c32k):
    cfg, x = c32k
    out, idx = run_prefill(cfg, x)
    L = cfg.L
    rows = np.unique(np.concatenate([[0, 1, cfg.k - 2, cfg.k - 1, cfg.k, 255, 256, 4095, 4096, L - 257, L - 1],
                                     synth.sample_rows(21, L, seed=1)]))
    mm = check_prefill(cfg, x, idx.cpu().numpy()[rows], bf16_tensor_to_f64(out[torch.from_numpy(rows).cuda()]),
                       rows)
    # idx rows of short prefixes hold every causal key
    got = idx[:cfg.k].cpu().numpy()
    for t in (0, 7, cfg.k - 1):
        assert sorted(got[t][got[t] >= 0].tolist()) == list(range(t + 1))
    print("32k index mismatch stats", mm)


def test_prefill_32k_deterministic(cuda_ok, c32k):
    cfg, x = c32k
    out1, idx1 = run_prefill(cfg, x)
    out2, idx2 = run_prefill(cfg, x, ws_bytes=3000 * cfg.L * 4)       # several chunks
    assert torch.equal(idx1, idx2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def make_decode_case(B, Lmax, ctx, steps, seed_cfg="32k"):
    """Sequences of the 32k workload's layout; ctx[b] tokens cached, `steps` new tokens each."""
    cfg = synth.CONFIGS[seed_cfg]
    data = [synth.inputs(cfg, 0, int(ctx[b]) + steps, seq=b) for b in range(B)]
    kc = np.zeros((B, Lmax, cfg.Hkv, cfg.D), dtype=np.uint16)
    vc = np.zeros_like(kc)
    kIc = np.zeros((B, Lmax, cfg.dI), dtype=np.uint16)
    for b in range(B):
        c = int(ctx[b])
        kc[b, :c], vc[b, :c], kIc[b, :c] = data[b]["k"][:c], data[b]["v"][:c], data[b]["kI"][:c]
    return cfg, data, kc, vc, kIc


def test_decode_steps_against_oracle(cuda_ok):
    B, Lmax, steps = 4, 6144, 3
    ctx = np.array([5, 1500, 2047, 6000])
    cfg, data, kc, vc, kIc = make_decode_case(B, Lmax, ctx, steps)
    kc_t, vc_t, kIc_t = dev(kc), dev(vc), dev(kIc)
    ctx_t = torch.from_numpy(ctx.astype(np.int32)).cuda()
    out = torch.empty((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
    for j in range(steps):
        pos = ctx + j
        sel = lambda name: np.stack([data[b][name][pos[b]] for b in range(B)])  # noqa: E731
        dsa.dsa_decode(dev(sel("q")), dev(sel("qI")), dev(sel("w")), dev(sel("k")), dev(sel("v")), dev(sel("kI")),
                       kc_t, vc_t, kIc_t, ctx_t, cfg.k, cfg.scale, out, idx, update_ctx=True)
        assert dsa.sync_status() == dsa.DSA_OK
        assert np.array_equal(ctx_t.cpu().numpy(), pos + 1)
        got_idx, got_out = idx.cpu().numpy(), bf16_tensor_to_f64(out)
        for b in range(B):
            t = int(pos[b])
            d = data[b]
            r = np.array([t])
            ref = oracle.dsa_rows(d["q"][r], d["qI"][r], d["w"][r], d["k"], d["v"], d["kI"], r, cfg.k, cfg.scale,
                                  keep_scores=True)
            mm = index_set_mismatch(got_idx[b:b + 1], ref["idx"], ref["scores"], ref["tau"], ref["absmax"], r + 1)
            assert mm["structural"] == 0 and mm["out_of_band"] == 0, (b, j, mm)
            own, _ = oracle.sparse_attn_rows(d["q"][r], d["k"], d["v"], got_idx[b:b + 1], cfg.scale)
            assert_output_ok(got_out[b:b + 1], own, f"decode b={b} step={j}")


def test_decode_many_sequences_one_cta_per_token(cuda_ok):
    """Enough sequences that the attention runs one CTA per token (no key splits): the new rows
    land in the caches, every context length advances by one, and sampled sequences match the
    oracle; one sequence has a context longer than k so its top-k is a real selection."""
    B, Lmax, steps = 300, 2200, 2
    rng = np.random.default_rng(15)
    ctx = rng.integers(1, 400, size=B)
    ctx[7] = 2100
    cfg, data, kc, vc, kIc = make_decode_case(B, Lmax, ctx, steps)
    kc_t, vc_t, kIc_t = dev(kc), dev(vc), dev(kIc)
    ctx_t = torch.from_numpy(ctx.astype(np.int32)).cuda()
    out = torch.empty((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, cfg.k), dtype=torch.int32, device="cuda")
    for j in range(steps):
        pos = ctx + j
        sel = lambda name: np.stack([data[b][name][pos[b]] for b in range(B)])  # noqa: E731
        dsa.dsa_decode(dev(sel("q")), dev(sel("qI")), dev(sel("w")), dev(sel("k")), dev(sel("v")), dev(sel("kI")),
                       kc_t, vc_t, kIc_t, ctx_t, cfg.k, cfg.scale, out, idx, update_ctx=True)
        assert dsa.sync_status() == dsa.DSA_OK
        assert np.array_equal(ctx_t.cpu().numpy(), pos + 1)
        for b in (0, 7, 100, B - 1):
            row = lambda c: c[b, int(pos[b])].view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
            assert np.array_equal(row(kc_t), data[b]["k"][pos[b]])
            assert np.array_equal(row(vc_t), data[b]["v"][pos[b]])
            assert np.array_equal(row(kIc_t), data[b]["kI"][pos[b]])
        got_idx, got_out = idx.cpu().numpy(), bf16_tensor_to_f64(out)
        for b in (0, 7, 100, B - 1):
            t = int(pos[b])
            d = data[b]
            r = np.array([t])
            ref = oracle.dsa_rows(d["q"][r], d["qI"][r], d["w"][r], d["k"], d["v"], d["kI"], r, cfg.k, cfg.scale,
                                  keep_scores=True)
            mm = index_set_mismatch(got_idx[b:b + 1], ref["idx"], ref["scores"], ref["tau"], ref["absmax"], r + 1)
            assert mm["structural"] == 0 and mm["out_of_band"] == 0, (b, j, mm)
            own, _ = oracle.sparse_attn_rows(d["q"][r], d["k"], d["v"], got_idx[b:b + 1], cfg.scale)
            assert_output_ok(got_out[b:b + 1], own, f"decode b={b} step={j}")


def test_decode_matches_prefill_row(cuda_ok):
    """A decode step at position t gives the prefill result of row t: the same index set except
    keys inside the near-tie band (the decode and prefill indexers round differently within fp32
    accuracy), and a close output."""
    cfg = synth.CONFIGS["32k"]
    L = 3000
    x = synth.inputs(cfg, 0, L)
    sub = synth.Config("sub", cfg.cid, L, cfg.k, layout=cfg.layout, p0=cfg.p0)
    out_p, idx_p = run_prefill(sub, x)
    Lmax, t = 3072, L - 1
    kc = np.zeros((1, Lmax, cfg.Hkv, cfg.D), dtype=np.uint16)
    vc, kIc = np.zeros_like(kc), np.zeros((1, Lmax, cfg.dI), dtype=np.uint16)
    kc[0, :t], vc[0, :t], kIc[0, :t] = x["k"][:t], x["v"][:t], x["kI"][:t]
    ctx = torch.tensor([t], dtype=torch.int32, device="cuda")
    out = torch.empty((1, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device="cuda")
    dsa.dsa_decode(dev(x["q"][t:t + 1]), dev(x["qI"][t:t + 1]), dev(x["w"][t:t + 1]), dev(x["k"][t:t + 1]),
                   dev(x["v"][t:t + 1]), dev(x["kI"][t:t + 1]), dev(kc), dev(vc), dev(kIc), ctx, cfg.k, cfg.scale,
                   out, idx)
    assert dsa.sync_status() == dsa.DSA_OK
    r = np.array([t])
    ref = oracle.dsa_rows(x["q"][r], x["qI"][r], x["w"][r], x["k"], x["v"], x["kI"], r, cfg.k, cfg.scale,
                          keep_scores=True)
    gd, gp = idx.cpu().numpy(), idx_p[t:t + 1].cpu().numpy()
    for got in (gd, gp):
        mm = index_set_mismatch(got, ref["idx"], ref["scores"], ref["tau"], ref["absmax"], r + 1)
        assert mm["structural"] == 0 and mm["out_of_band"] == 0, mm
    sym = np.setxor1d(gd[0], gp[0])
    band = 1e-3 * abs(ref["tau"][0]) + 1e-6 * ref["absmax"][0]
    assert np.all(np.abs(ref["scores"][0, sym] - ref["tau"][0]) <= band), sym
    if len(sym) == 0:
        d = (out[0].double() - out_p[t].double()).abs().max().item()
        assert d <= 1e-2


def test_decode_bad_context_length_reports_error(cuda_ok):
    B, Lmax = 2, 1024
    cfg = synth.CONFIGS["32k"]
    kc = torch.zeros((B, Lmax, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kIc = torch.zeros((B, Lmax, cfg.dI), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    qI = torch.zeros((B, cfg.HI, cfg.dI), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((B, cfg.HI), dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros((B, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device="cuda")
    kIn = torch.zeros((B, cfg.dI), dtype=torch.bfloat16, device="cuda")
    ctx = torch.tensor([10, Lmax + 5], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    dsa.dsa_decode(q, qI, w, kn, kn, kIn, kc, vc, kIc, ctx, 256, 0.1, out)
    assert dsa.sync_status() == dsa.DSA_ERR_DEVICE_INPUT
    assert dsa.sync_status() == dsa.DSA_OK          # the error word was cleared
    torch.cuda.synchronize()


def test_bounded_wait_timeout_reports_and_context_survives(cuda_ok):
    dsa.selftest_timeout(50_000_000)                # 50 ms wait on a barrier nobody completes
    assert dsa.sync_status() == dsa.DSA_ERR_TIMEOUT
    assert dsa.sync_status() == dsa.DSA_OK
    x = torch.ones(1000, device="cuda")             # the context is still usable
    assert float(x.sum()) == 1000.0


def test_profile_and_launch_counter(cuda_ok, tiny):
    cfg, x, _ = tiny
    n0 = dsa.launch_count()
    dsa.profile_begin()
    run_prefill(cfg, x)
    prof = dsa.profile_end()
    assert dsa.launch_count() - n0 == 3
    assert prof["indexer"]["launches"] == 1 and prof["topk"]["launches"] == 1 and prof["sparse_attn"]["launches"] == 1
    assert all(v["ms"] > 0 for k, v in prof.items() if v["launches"])


@pytest.mark.parametrize("W", [1, 100, 3000])
def test_topk_window_exact_on_oracle_scores(cuda_ok, tiny, W):
    """Sliding-window top-k (SW-DSA) on the oracle's fp32 scores equals the oracle's, exactly."""
    cfg, x, ref = tiny
    L = cfg.L
    s32 = np.nan_to_num(ref["scores"], nan=0.0).astype(np.float32)
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(torch.from_numpy(s32).cuda(), 0, cfg.k, idx, window=W)
    assert dsa.sync_status() == dsa.DSA_OK
    want, _ = oracle.topk_rows(s32.astype(np.float64), np.arange(L) + 1, cfg.k, window=W)
    got = idx.cpu().numpy()
    for r in range(L):
        assert sorted(got[r].tolist()) == sorted(want[r].tolist()), r


@pytest.mark.parametrize("name,W", [("tiny", 300), ("32k", 4096), ("32k", 40000)])
def test_prefill_window_sampled_rows(cuda_ok, name, W):
    cfg = synth.CONFIGS[name]
    x = synth.inputs(cfg, 0, cfg.L)
    L = cfg.L
    out = torch.empty((L, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
    d = {n: dev(a) for n, a in x.items()}
    dsa.dsa_prefill(d["q"], d["k"], d["v"], d["qI"], d["kI"], d["w"], cfg.k, cfg.scale, out, idx, window=W)
    assert dsa.sync_status() == dsa.DSA_OK
    rows = np.unique(np.concatenate([[0, W - 2, W - 1, W, W + 1, L - 1], synth.sample_rows(13, L, seed=5)]))
    rows = rows[(rows >= 0) & (rows < L)]
    ref = oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows, cfg.k,
                          cfg.scale, keep_scores=True, window=W)
    gi = idx.cpu().numpy()[rows]
    n_win = np.minimum(rows + 1, W)
    for r, t in enumerate(rows):                       # every selected key inside the window
        sel = gi[r][gi[r] >= 0]
        assert len(sel) == min(cfg.k, n_win[r]) and sel.min() >= t - W + 1 and sel.max() <= t
    mm = index_set_mismatch(gi, ref["idx"], ref["scores"], ref["tau"], ref["absmax"], rows + 1)
    assert mm["out_of_band"] == 0, mm
    own, _ = oracle.sparse_attn_rows(x["q"][rows], x["k"], x["v"], gi, cfg.scale)
    assert_output_ok(bf16_tensor_to_f64(out[torch.from_numpy(rows).cuda()]), own, f"window {W}")


def test_sparse_attn_random_gather_beyond_l2(cuda_ok):
    """K/V far larger than L2 (2 x 268 MB) and uniformly random indices: most row copies miss L2
    and land out of order, the case in which a pipeline that confused barrier phases would read
    a stage before its copies arrived (or stall)."""
    g = torch.Generator().manual_seed(14)
    Lk, T, Hq, Hkv, topk = 262144, 4096, 32, 4, 2048
    q0 = Lk - T
    tq = torch.randn((T, Hq, 128), generator=g).to(torch.bfloat16)
    tk = torch.randn((Lk, Hkv, 128), generator=g).to(torch.bfloat16)
    tv = torch.randn((Lk, Hkv, 128), generator=g).to(torch.bfloat16)
    t_abs = torch.arange(q0, Lk, dtype=torch.int64)
    idx = (torch.rand((T, topk), generator=g, dtype=torch.float64) * (t_abs[:, None] + 1).double()).long()
    idx = idx.clamp_max(t_abs[:, None]).to(torch.int32)
    out = torch.empty((T, Hq, 128), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        dsa.dsa_sparse_attn(tq.cuda(), tk.cuda(), tv.cuda(), idx.cuda(), q0, 0.0883883, out)
        assert dsa.sync_status() == dsa.DSA_OK
    rows = np.linspace(0, T - 1, 48).astype(np.int64)
    bits = [t.view(torch.int16).numpy().view(np.uint16) for t in (tq, tk, tv)]
    want, _ = oracle.sparse_attn_rows(bits[0][rows], bits[1], bits[2], idx.numpy()[rows], 0.0883883)
    assert_output_ok(bf16_tensor_to_f64(out)[rows], want, "random gather")


def test_attention_skips_padding_entries_inside_the_count(cuda_ok):
    """Entries that name no key (-1, or >= Lk) are skipped wherever they sit in the list."""
    rng = np.random.default_rng(13)
    L, Hq, Hkv, topk = 300, 8, 2, 64
    tq, tk, tv = (torch.from_numpy(rng.standard_normal(sh).astype(np.float32)).to(torch.bfloat16)
                  for sh in ((L, Hq, 128), (L, Hkv, 128), (L, Hkv, 128)))
    bits = [t.view(torch.int16).numpy().view(np.uint16) for t in (tq, tk, tv)]
    idx = np.full((L, topk), -1, dtype=np.int32)
    for t in range(L):
        m = min(topk, t + 1)
        idx[t, :m] = rng.choice(t + 1, size=m, replace=False)
        holes = rng.choice(m, size=m // 4, replace=False)
        idx[t, holes[: len(holes) // 2]] = -1
        idx[t, holes[len(holes) // 2:]] = L + 7            # out of range
    out = torch.empty((L, Hq, 128), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_sparse_attn(tq.cuda(), tk.cuda(), tv.cuda(), torch.from_numpy(idx).cuda(), 0, 0.0883883, out)
    assert dsa.sync_status() == dsa.DSA_OK
    clean = np.where(idx >= L, -1, idx).astype(np.int32)
    want, _ = oracle.sparse_attn_rows(bits[0], bits[1], bits[2], clean, 0.0883883)
    assert_output_ok(bf16_tensor_to_f64(out), want, "holes")


def test_prefill_rows_ranges_reproduce_prefill(cuda_ok, c32k):
    """Consecutive row ranges through dsa_prefill_rows (row-local q/qI/w/out) give exactly the
    indices and outputs of one dsa_prefill over the whole sequence."""
    cfg, x = c32k
    out_full, idx_full = run_prefill(cfg, x)
    d = {n: dev(a) for n, a in x.items()}
    out = torch.empty_like(out_full)
    idx = torch.empty_like(idx_full)
    for r0, r1 in ((0, 777), (777, 9000), (9000, 20001), (20001, cfg.L)):
        dsa.dsa_prefill_rows(d["q"][r0:r1], d["k"][:r1], d["v"][:r1], d["qI"][r0:r1], d["kI"][:r1], d["w"][r0:r1],
                             r0, cfg.k, cfg.scale, out[r0:r1], idx[r0:r1])
    assert dsa.sync_status() == dsa.DSA_OK
    assert torch.equal(idx, idx_full)
    assert torch.equal(out.view(torch.int16), out_full.view(torch.int16))


# ----------------------------------------------------------------------------- warm-up KL target
# Tolerance: logits are fp32 sums of 128 exact bf16 products, P and log P come from fp32
# exp2/log2 (a few ulp) and per-lane fp32 sums over <= 32K keys, and the indexer scores carry
# their own fp32 error, which enters KL linearly (sum_s P_t(s) * dscore).  Together well below
# 1e-4 relative on these inputs; the test allows 2e-4 + 2e-4 |KL|.
KL_ATOL, KL_RTOL = 2e-4, 2e-4


def run_kl(x, L, scale, ws_bytes=None):
    kl = torch.empty(L, dtype=torch.float32, device="cuda")
    ws = None if ws_bytes is None else torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    dsa.dsa_indexer_kl(dev(x["q"][:L]), dev(x["k"][:L]), dev(x["qI"][:L]), dev(x["kI"][:L]), dev(x["w"][:L]), scale,
                       kl, ws)
    assert dsa.sync_status() == dsa.DSA_OK
    return kl.cpu().numpy().astype(np.float64)


def test_indexer_kl_tiny_every_row(cuda_ok, tiny):
    cfg, x, _ = tiny
    got = run_kl(x, cfg.L, cfg.scale)
    rows = np.arange(cfg.L)
    want = oracle.kl_rows(x["q"], x["k"], x["qI"], x["w"], x["kI"], rows, cfg.scale)
    np.testing.assert_allclose(got, want, rtol=KL_RTOL, atol=KL_ATOL)
    assert got[0] == pytest.approx(0.0, abs=1e-6)


def test_indexer_kl_32k_sampled_rows_and_chunking(cuda_ok, c32k):
    cfg, x = c32k[0], c32k[1]
    L = 6000
    got = run_kl(x, L, cfg.scale)
    rows = np.array([0, 1, 15, 16, 17, 255, 256, 2047, 2048, 4099, L - 2, L - 1])
    want = oracle.kl_rows(x["q"][rows], x["k"], x["qI"][rows], x["w"][rows], x["kI"], rows, cfg.scale)
    np.testing.assert_allclose(got[rows], want, rtol=KL_RTOL, atol=KL_ATOL)
    assert np.all(np.isfinite(got)) and np.all(got > -KL_ATOL)
    # a workspace of 1000 score rows: six chunks, the same values bit for bit
    small = run_kl(x, L, cfg.scale, ws_bytes=1000 * ((L + 3) // 4 * 4) * 4 + 512)
    assert np.array_equal(small, got)


def test_indexer_kl_gqa_shapes(cuda_ok):
    rng = np.random.default_rng(16)
    L, HI, dI = 500, 8, 64
    for Hq, Hkv in ((16, 2), (8, 4), (8, 1)):
        q, k = rng.standard_normal((L, Hq, 128)), rng.standard_normal((L, Hkv, 128))
        qI, kI, w = rng.standard_normal((L, HI, dI)), rng.standard_normal((L, dI)), rng.standard_normal((L, HI))
        tq, tk, tqI, tkI, tw = (torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16) for a in (q, k, qI, kI, w))
        bits = [t.view(torch.int16).numpy().view(np.uint16) for t in (tq, tk, tqI, tkI, tw)]
        kl = torch.empty(L, dtype=torch.float32, device="cuda")
        dsa.dsa_indexer_kl(tq.cuda(), tk.cuda(), tqI.cuda(), tkI.cuda(), tw.cuda(), 0.0883883, kl)
        assert dsa.sync_status() == dsa.DSA_OK
        want = oracle.kl_rows(bits[0], bits[1], bits[2], bits[4], bits[3], np.arange(L), 0.0883883)
        np.testing.assert_allclose(kl.cpu().numpy().astype(np.float64), want, rtol=KL_RTOL, atol=KL_ATOL,
                                   err_msg=f"Hq={Hq} Hkv={Hkv}")


def canonical_order(selected, n_comp, lo, k):
    """The documented output order of a top-k row: ascending when every competing key is kept,
    else grouped by region ((index / 32) mod 4) and ascending within a region; -1 padding."""
    sel = [int(i) for i in selected if i >= 0]
    if n_comp <= k:
        row = list(range(lo, lo + n_comp))
    else:
        row = sorted(sel, key=lambda i: ((i // 32) % 4, i))
    return row + [-1] * (k - len(row))


def test_topk_randomized_exact_order(cuda_ok):
    """Random row lengths, k, windows and score distributions (Gaussian, heavy integer ties,
    signed zeros): the GPU rows equal the oracle's sets in the documented order, entry by entry."""
    rng = np.random.default_rng(17)
    for case in range(18):
        rows = int(rng.integers(1, 24))
        q_pos0 = int(rng.integers(0, 20000))
        k = int(rng.choice([1, 7, 64, 300, 2048, 4096]))
        window = int(rng.choice([0, 0, 100, 5000]))
        n_max = q_pos0 + rows
        ld = (n_max + 3) // 4 * 4
        kind = case % 3
        if kind == 0:
            s = (rng.standard_normal((rows, ld)) * 10).astype(np.float32)
        elif kind == 1:
            s = rng.integers(-2, 3, size=(rows, ld)).astype(np.float32)
        else:
            s = np.where(rng.random((rows, ld)) < 0.5, np.float32(0.0), np.float32(-0.0))
            s[:, ::13] = 2.0
        idx = torch.empty((rows, k), dtype=torch.int32, device="cuda")
        dsa.dsa_topk(torch.from_numpy(s).cuda(), q_pos0, k, idx, window=window)
        assert dsa.sync_status() == dsa.DSA_OK
        n = q_pos0 + np.arange(rows) + 1
        want, _ = oracle.topk_rows(s.astype(np.float64), n, k, window=window)
        got = idx.cpu().numpy()
        for r in range(rows):
            lo = max(0, int(n[r]) - window) if window > 0 else 0
            expect = canonical_order(want[r], int(n[r]) - lo, lo, k)
            assert got[r].tolist() == expect, (case, r, rows, q_pos0, k, window, kind)


def test_indexer_kl_short_and_ragged_sequences(cuda_ok, tiny):
    """L = 1 (KL 0), L < 8 and L not a multiple of the 8-token blocks."""
    cfg, x, _ = tiny
    for L in (1, 5, 13, 100):
        got = run_kl(x, L, cfg.scale)
        want = oracle.kl_rows(x["q"][:L], x["k"], x["qI"][:L], x["w"][:L], x["kI"], np.arange(L), cfg.scale)
        np.testing.assert_allclose(got, want, rtol=KL_RTOL, atol=KL_ATOL, err_msg=f"L={L}")


@pytest.mark.parametrize("HI", [1, 2, 8, 16, 64])
def test_index_every_head_count(cuda_ok, HI):
    """Every supported indexer head count (its own kernel instantiation: HI = 64 spans two
    accumulator chunks per token, HI < 4 has no ReLU pipe split): a ragged slice of a causal
    sequence against the oracle, within the fp32 bound, nothing written past the diagonal."""
    rng = np.random.default_rng(18 + HI)
    q_pos0, Lq, dI = 700, 333, 64
    Lk = q_pos0 + Lq
    tqI, tkI, tw = (torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
                    for a in (rng.standard_normal((Lq, HI, dI)), rng.standard_normal((Lk, dI)),
                              rng.standard_normal((Lq, HI))))
    qI, kI, w = (t.view(torch.int16).numpy().view(np.uint16) for t in (tqI, tkI, tw))
    ld = (Lk + 3) // 4 * 4
    scores = torch.full((Lq, ld), float("nan"), device="cuda")
    dsa.dsa_index(tqI.cuda(), tkI.cuda(), tw.cuda(), q_pos0, scores)
    assert dsa.sync_status() == dsa.DSA_OK
    rows = np.arange(q_pos0, q_pos0 + Lq)
    ref = oracle.index_rows(qI, w, kI, rows)
    got = scores.cpu().double().numpy()[:, :Lk]
    bound = 1e-5 * score_bound(qI, w, kI, rows) + 1e-30
    for r in range(Lq):
        n = rows[r] + 1
        assert np.all(np.abs(got[r, :n] - ref[r, :n]) <= bound[r, :n]), (HI, r)
        assert np.all(np.isnan(got[r, n:]))


def test_decode_sixteen_heads_per_kv_group(cuda_ok):
    """Decode with Hq = 32 over Hkv = 2 (16 heads per group: two 8-head MMA tiles, with key
    splits and the merge) and HI = 16, against the oracle on every sequence."""
    rng = np.random.default_rng(19)
    B, Lmax, Hq, Hkv, D, HI, dI, topk, scale = 3, 3000, 32, 2, 128, 16, 64, 512, 0.0883883
    ctx = np.array([10, 700, 2900])
    f = lambda *sh: torch.from_numpy(rng.standard_normal(sh).astype(np.float32)).to(torch.bfloat16)  # noqa: E731
    kc, vc, kIc = f(B, Lmax, Hkv, D), f(B, Lmax, Hkv, D), f(B, Lmax, dI)
    q, qI, w = f(B, Hq, D), f(B, HI, dI), f(B, HI)
    kn, vn, kIn = f(B, Hkv, D), f(B, Hkv, D), f(B, dI)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    ctx_t = torch.from_numpy(ctx.astype(np.int32)).cuda()
    kc_d, vc_d, kIc_d = kc.cuda(), vc.cuda(), kIc.cuda()
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, topk), dtype=torch.int32, device="cuda")
    dsa.dsa_decode(q.cuda(), qI.cuda(), w.cuda(), kn.cuda(), vn.cuda(), kIn.cuda(), kc_d, vc_d, kIc_d, ctx_t, topk,
                   scale, out, idx, update_ctx=True)
    assert dsa.sync_status() == dsa.DSA_OK
    assert np.array_equal(ctx_t.cpu().numpy(), ctx + 1)
    got_idx, got_out = idx.cpu().numpy(), bf16_tensor_to_f64(out)
    for b in range(B):
        t = int(ctx[b])
        k_all, v_all, kI_all = bits(kc[b]).copy(), bits(vc[b]).copy(), bits(kIc[b]).copy()
        k_all[t], v_all[t], kI_all[t] = bits(kn[b]), bits(vn[b]), bits(kIn[b])
        r = np.array([t])
        ref = oracle.dsa_rows(bits(q[b:b + 1]), bits(qI[b:b + 1]), bits(w[b:b + 1]), k_all, v_all, kI_all, r, topk,
                              scale, keep_scores=True)
        mm = index_set_mismatch(got_idx[b:b + 1], ref["idx"], ref["scores"], ref["tau"], ref["absmax"], r + 1)
        assert mm["structural"] == 0 and mm["out_of_band"] == 0, (b, mm)
        own, _ = oracle.sparse_attn_rows(bits(q[b:b + 1]), k_all, v_all, got_idx[b:b + 1], scale)
        assert_output_ok(got_out[b:b + 1], own, f"decode G=16 b={b}")


@pytest.mark.parametrize("kind,k,window", [("gauss", 2048, 0), ("gauss", 300, 0), ("ties", 2048, 0),
                                           ("zeros", 2048, 0), ("gauss", 2048, 20000), ("frames", 2048, 0),
                                           ("gauss", 4096, 0), ("decoy", 2048, 0)])
def test_topk_many_long_rows_exact_order(cuda_ok, kind, k, window):
    """A launch of many long rows (more than one per SM, as a prefill chunk) through the one-CTA
    kernel (the path counter proves it): every row equals the oracle's set in the documented
    order, entry by entry.  Gaussian scores, frame-correlated scores, heavy integer ties (the
    re-aimed second pass and the exact fallback), signed zeros, a sliding window, k at the
    candidate capacity, and decoys (raised scores at a regular stride of 4-key groups, a pattern
    that biases the sampled threshold)."""
    rng = np.random.default_rng(23 + k + window)
    rows, q_pos0 = 400, 60000 if kind == "decoy" else 30000
    n_max = q_pos0 + rows
    ld = (n_max + 3) // 4 * 4
    if kind == "gauss":
        s = (rng.standard_normal((rows, ld)) * 10).astype(np.float32)
    elif kind == "frames":                     # blocks of 512 keys sharing an offset
        s = (rng.standard_normal((rows, ld)) + np.repeat(rng.standard_normal((rows, ld // 512 + 1)) * 3, 512,
                                                         axis=1)[:, :ld]).astype(np.float32)
    elif kind == "ties":
        s = rng.integers(-2, 3, size=(rows, ld)).astype(np.float32)
    elif kind == "decoy":
        s = rng.standard_normal((rows, ld)).astype(np.float32)
        g = np.arange(ld // 4)
        s.reshape(rows, -1, 4)[:, g % 14 == 0, :] += 40.0
    else:
        s = np.where(rng.random((rows, ld)) < 0.5, np.float32(0.0), np.float32(-0.0))
        s[:, ::13] = 2.0
    idx = torch.full((rows, k), -5, dtype=torch.int32, device="cuda")
    dsa.read_counters(reset=True)
    dsa.dsa_topk(torch.from_numpy(s).cuda(), q_pos0, k, idx, window=window)
    assert dsa.sync_status() == dsa.DSA_OK
    cnt = dsa.read_counters(reset=True)
    assert cnt["topk_rows"] == rows and cnt["topk_cluster_rows"] == 0, cnt
    n = q_pos0 + np.arange(rows) + 1
    want, _ = oracle.topk_rows(s.astype(np.float64), n, k, window=window)
    got = idx.cpu().numpy()
    for r in range(rows):
        lo = max(0, int(n[r]) - window) if window > 0 else 0
        expect = canonical_order(want[r], int(n[r]) - lo, lo, k)
        assert got[r].tolist() == expect, (kind, k, window, r)
    if kind in ("ties", "zeros"):
        assert cnt["topk_retry"] > 0 and cnt["topk_global"] > 0   # both fallback passes ran


def test_topk_cluster_and_one_cta_kernels_agree(cuda_ok):
    """The same long rows through the one-CTA kernel (a launch of many rows) and the cluster
    kernel (a few rows per launch, 8 CTAs each) give identical outputs, entry by entry."""
    rng = np.random.default_rng(29)
    rows, q_pos0, k = 300, 40000, 2048
    ld = (q_pos0 + rows + 3) // 4 * 4
    s = torch.from_numpy((rng.standard_normal((rows, ld)) * 5).astype(np.float32)).cuda()
    a = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    b = torch.empty_like(a)
    dsa.read_counters(reset=True)
    dsa.dsa_topk(s, q_pos0, k, a)
    for r0 in range(0, rows, 12):                        # 12 rows x 8 CTAs <= 2 per SM: clusters
        dsa.dsa_topk(s[r0:r0 + 12], q_pos0 + r0, k, b[r0:r0 + 12])
    assert dsa.sync_status() == dsa.DSA_OK
    cnt = dsa.read_counters(reset=True)
    assert cnt["topk_rows"] == rows and cnt["topk_cluster_rows"] == rows, cnt
    assert torch.equal(a, b)


@pytest.mark.parametrize("n,kind", [(300_000, "gauss"), (300_000, "ties"), (400_000, "gauss")])
def test_topk_cluster_staged_and_unstaged_segments(cuda_ok, n, kind):
    """The cluster kernel copies each CTA's eighth of a row into shared memory when it fits the
    stage (300K keys: 147 KB per CTA) and streams it from global memory when it does not (400K
    keys).  Both forms, and the exact fallback over the whole row (integer ties), give the
    oracle's set in the documented order, entry by entry."""
    rng = np.random.default_rng(31 + n)
    rows, k = 3, 2048
    q_pos0 = n - rows
    ld = (n + 3) // 4 * 4
    if kind == "ties":
        s = rng.integers(-2, 3, size=(rows, ld)).astype(np.float32)
    else:
        s = (rng.standard_normal((rows, ld)) * 7).astype(np.float32)
    idx = torch.full((rows, k), -5, dtype=torch.int32, device="cuda")
    dsa.read_counters(reset=True)
    dsa.dsa_topk(torch.from_numpy(s).cuda(), q_pos0, k, idx)
    assert dsa.sync_status() == dsa.DSA_OK
    cnt = dsa.read_counters(reset=True)
    assert cnt["topk_cluster_rows"] == rows and cnt["topk_rows"] == 0, cnt
    n_r = q_pos0 + np.arange(rows) + 1
    want, _ = oracle.topk_rows(s.astype(np.float64), n_r, k)
    got = idx.cpu().numpy()
    for r in range(rows):
        assert got[r].tolist() == canonical_order(want[r], int(n_r[r]), 0, k), (n, kind, r)
    if kind == "ties":
        assert cnt["topk_cluster_global"] > 0
