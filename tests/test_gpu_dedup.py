"""GPU parity of the adjacent-query dedup attention (dsa_sparse_attn_dedup) against the fp64 oracle
and against the per-token kernel, through the C ABI.

The dedup kernel computes each token's softmax over its own selected keys, so the oracle's
per-token sparse attention is the reference; tolerances are those of tests/parity.py.  Row orders
cover the ones the kernel treats differently: ascending rows (one run), rows in dsa_topk's region
order (four ascending runs), and rows in random order (more than 8 runs: whole-row scans).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_output_ok, bf16_tensor_to_f64

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("dsa_lightning_indexer_02_b200")

SCALE = 0.0883883


def _bf16(a):
    t = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    return t, t.view(torch.int16).numpy().view(np.uint16)


def _order(sel, order, rng):
    if order == "sorted":
        return np.sort(sel)
    if order == "regions":  # dsa_topk's order: grouped by (index / 32) mod 4, ascending within a group
        return sel[np.lexsort((sel, (sel // 32) % 4))]
    return rng.permutation(sel)


def make_case(Hq, Hkv, L, topk, order, seed, overlap=0.0, q_pos0=0, holes=False):
    """Queries of rows q_pos0 .. q_pos0+L-1 over keys 0 .. q_pos0+L-1.  overlap > 0: adjacent rows
    pick their keys by a shared key score plus per-row noise (so neighbours share most keys)."""
    rng = np.random.default_rng(seed)
    Lk = q_pos0 + L
    q = rng.standard_normal((L, Hq, 128))
    k = rng.standard_normal((Lk, Hkv, 128))
    v = rng.standard_normal((Lk, Hkv, 128))
    base = rng.standard_normal(Lk)
    idx = np.full((L, topk), -1, dtype=np.int32)
    for i in range(L):
        n_keys = q_pos0 + i + 1
        n = min(topk, n_keys)
        if overlap > 0:
            s = overlap * base[:n_keys] + rng.standard_normal(n_keys)
            sel = np.argsort(-s, kind="stable")[:n]
        else:
            sel = rng.choice(n_keys, size=n, replace=False)
        sel = _order(sel.astype(np.int32), order, rng)
        if holes and n > 4:
            sel[1] = -1
            sel[n // 2] = Lk + 5  # names no key: skipped
        idx[i, :n] = sel
    return q, k, v, idx


def run_both(q, k, v, idx, q_pos0):
    (tq, qb), (tk, kb), (tv, vb) = _bf16(q), _bf16(k), _bf16(v)
    L, Hq, D = q.shape
    dev = {n: t.cuda() for n, t in (("q", tq), ("k", tk), ("v", tv))}
    ti = torch.from_numpy(idx).cuda()
    out_d = torch.empty((L, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse_d = torch.empty((L, Hq), dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_attn_dedup(dev["q"], dev["k"], dev["v"], ti, q_pos0, SCALE, out_d, lse_d)
    st = dsa.sync_status()
    assert st == dsa.DSA_OK, (st, hex(dsa.error_site()))
    out_t = torch.empty_like(out_d)
    lse_t = torch.empty_like(lse_d)
    dsa.dsa_sparse_attn(dev["q"], dev["k"], dev["v"], ti, q_pos0, SCALE, out_t, lse_t)
    assert dsa.sync_status() == dsa.DSA_OK
    return (qb, kb, vb), (out_d, lse_d), (out_t, lse_t)


def oracle_idx(idx, n_keys):
    return np.where((idx < 0) | (idx >= n_keys), -1, idx).astype(np.int32)


@pytest.mark.parametrize("Hq,Hkv,L,topk,order,overlap,holes", [
    (16, 2, 700, 300, "random", 0.0, False),    # G = 8, 16 tokens per block, whole-row scans
    (16, 2, 700, 300, "sorted", 3.0, False),    # one run per row, neighbours overlapping
    (32, 4, 517, 256, "regions", 3.0, True),    # top-k order, holes and out-of-range entries
    (32, 2, 300, 128, "regions", 0.0, False),   # G = 16, 8 tokens per block
    (8, 1, 1100, 1024, "sorted", 0.0, False),   # a row of the union spans several windows
])
def test_dedup_matches_oracle_and_per_token(cuda_ok, Hq, Hkv, L, topk, order, overlap, holes):
    q, k, v, idx = make_case(Hq, Hkv, L, topk, order, seed=L + topk, overlap=overlap, holes=holes)
    bits, (out_d, lse_d), (out_t, lse_t) = run_both(q, k, v, idx, 0)
    want, want_lse = oracle.sparse_attn_rows(bits[0], bits[1], bits[2], oracle_idx(idx, k.shape[0]), SCALE)
    assert_output_ok(bf16_tensor_to_f64(out_d), want, f"dedup {order}")
    assert_output_ok(bf16_tensor_to_f64(out_d), bf16_tensor_to_f64(out_t), "dedup vs per-token")
    np.testing.assert_allclose(lse_d.cpu().numpy(), want_lse, rtol=0, atol=2e-3)


def test_dedup_ragged_rows_and_offset(cuda_ok):
    """q_pos0 > 0 (a later chunk of rows) and a row count that leaves the last block partial."""
    q, k, v, idx = make_case(16, 2, 333, 200, "regions", seed=5, overlap=2.0, q_pos0=1000)
    bits, (out_d, lse_d), _ = run_both(q, k, v, idx, 1000)
    want, want_lse = oracle.sparse_attn_rows(bits[0], bits[1], bits[2], oracle_idx(idx, k.shape[0]), SCALE)
    assert_output_ok(bf16_tensor_to_f64(out_d), want, "dedup offset")
    np.testing.assert_allclose(lse_d.cpu().numpy(), want_lse, rtol=0, atol=2e-3)


def test_dedup_rows_without_keys(cuda_ok):
    """Rows whose every entry names no key give zeros and lse = -inf; the others are unaffected."""
    q, k, v, idx = make_case(16, 2, 64, 32, "sorted", seed=9)
    idx[5:21] = -1                      # one whole block of 16 rows without keys, and a partial one
    bits, (out_d, lse_d), _ = run_both(q, k, v, idx, 0)
    o = bf16_tensor_to_f64(out_d)
    assert np.all(o[5:21] == 0.0)
    assert np.all(np.isneginf(lse_d.cpu().numpy()[5:21]))
    keep = np.r_[0:5, 21:64]
    want, _ = oracle.sparse_attn_rows(bits[0][keep], bits[1], bits[2], oracle_idx(idx[keep], k.shape[0]), SCALE)
    assert_output_ok(o[keep], want, "dedup rows with keys")


def test_dedup_on_32k_topk_indices(cuda_ok):
    """The 32K workload's own top-k rows (dsa_prefill's indices): dedup output against the oracle
    on sampled rows and against the per-token kernel on every row."""
    cfg = synth.CONFIGS["32k"]
    x = synth.inputs(cfg, 0, cfg.L)
    d = {n: synth.to_torch(a).cuda() for n, a in x.items()}
    L = cfg.L
    out_t = torch.empty((L, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device="cuda")
    dsa.dsa_prefill(d["q"], d["k"], d["v"], d["qI"], d["kI"], d["w"], cfg.k, cfg.scale, out_t, idx)
    out_d = torch.empty_like(out_t)
    dsa.dsa_sparse_attn_dedup(d["q"], d["k"], d["v"], idx, 0, cfg.scale, out_d)
    assert dsa.sync_status() == dsa.DSA_OK
    assert_output_ok(bf16_tensor_to_f64(out_d), bf16_tensor_to_f64(out_t), "dedup vs per-token, every row")
    rows = np.unique(np.concatenate([[0, 1, 15, 16, 2047, 2048, L - 17, L - 1], synth.sample_rows(24, L, seed=3)]))
    gi = idx.cpu().numpy()[rows]
    want, _ = oracle.sparse_attn_rows(x["q"][rows], x["k"], x["v"], gi, cfg.scale)
    assert_output_ok(bf16_tensor_to_f64(out_d[torch.from_numpy(rows).cuda()]), want, "dedup vs oracle")
