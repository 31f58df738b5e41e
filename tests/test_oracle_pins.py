"""Pins of the fp64 CPU oracle against facts that do not come from the oracle itself.

Each test fixes one part of what the oracle computes by a closed form, a library special case,
brute force on a tiny input, or an invariant, chosen so that a plausible slip (a dropped ReLU,
a transposed operand, a wrong GQA head map, a reversed tie rule, a missing softmax scale)
fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def bf16_bits(x) -> np.ndarray:
    """float64 values that are exactly representable in bf16 -> bf16 bits."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.to(torch.float64), torch.as_tensor(np.asarray(x, dtype=np.float64)))
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_bf16(rng, shape, scale=1.0):
    x = torch.as_tensor(rng.standard_normal(shape) * scale, dtype=torch.float32).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def f64(bits):
    return synth.bf16_to_f64(bits)


# ----------------------------------------------------------------------------- indexer


def test_indexer_scaled_basis_keys_closed_form():
    """kI[s] = c_s * e_{j(s)}: q.k_s = c_s * qI[h, j(s)], so the scores follow by indexing."""
    rng = np.random.default_rng(1)
    HI, dI, L = 3, 8, 24
    j_of = rng.integers(0, dI, size=L)
    c_of = rng.choice([0.5, 1.0, 2.0, -1.0, -0.25], size=L)
    kI = np.zeros((L, dI))
    kI[np.arange(L), j_of] = c_of
    qI = rand_bf16(rng, (L, HI, dI))
    w = rand_bf16(rng, (L, HI))
    t_rows = np.arange(L)
    got = oracle.index_rows(qI, w, bf16_bits(kI), t_rows)
    qf, wf = f64(qI), f64(w)
    for t in range(L):
        for s in range(t + 1):
            dots = c_of[s] * qf[t, :, j_of[s]]          # one dot per head
            want = float(np.sum(wf[t] * np.maximum(dots, 0.0)))
            assert got[t, s] == pytest.approx(want, rel=0, abs=1e-12)
        assert np.all(np.isnan(got[t, t + 1:]))        # causal: nothing written beyond t


def test_indexer_single_head_unit_weight_is_relu_of_matmul():
    """H_I = 1, w = 1: score = ReLU(qI . kI), a plain matrix product (numpy) then clamp."""
    rng = np.random.default_rng(2)
    L, dI = 40, 64
    qI = rand_bf16(rng, (L, 1, dI))
    kI = rand_bf16(rng, (L, dI))
    w = bf16_bits(np.ones((L, 1)))
    got = oracle.index_rows(qI, w, kI, np.arange(L))
    want = np.maximum(f64(qI)[:, 0, :] @ f64(kI).T, 0.0)
    mask = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(got[mask], want[mask], rtol=1e-13, atol=1e-13)


def test_indexer_negative_weight_and_relu():
    """ReLU acts on each head's dot before weighting: one head with dot -5 contributes 0,
    another with dot +3 contributes w*3 even when w < 0."""
    dI = 4
    qI = bf16_bits([[[1, 0, 0, 0], [0, 1, 0, 0]]])            # head 0 picks d0, head 1 picks d1
    kI = bf16_bits([[-5, 3, 0, 0]])
    w = bf16_bits([[2.0, -0.5]])
    got = oracle.index_rows(qI, w, kI, [0])
    assert got[0, 0] == -1.5                                  # 2*relu(-5) + (-0.5)*relu(3)


def test_indexer_weight_scaling_invariance():
    """w -> 2w doubles every score exactly and leaves the top-k set unchanged."""
    rng = np.random.default_rng(3)
    L, HI, dI, k = 64, 4, 64, 16
    qI, kI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, dI)), rand_bf16(rng, (L, HI))
    w2 = bf16_bits(2.0 * f64(w))
    s1 = oracle.index_rows(qI, w, kI, np.arange(L))
    s2 = oracle.index_rows(qI, w2, kI, np.arange(L))
    mask = np.tril(np.ones((L, L), dtype=bool))
    assert np.array_equal(2.0 * s1[mask], s2[mask])
    i1, _ = oracle.topk_rows(np.nan_to_num(s1, nan=-np.inf), np.arange(L) + 1, k)
    i2, _ = oracle.topk_rows(np.nan_to_num(s2, nan=-np.inf), np.arange(L) + 1, k)
    assert np.array_equal(i1, i2)


def test_row_absmax_and_tau_on_a_designed_row():
    """dsa_rows reports, per row, absmax = max_s |score(t, s)| (the absolute floor of the parity
    band) and tau = the score of the last selected key.  Hand case: one head picking channel 0,
    keys with channel-0 values 1, 3, -4, 0.5: ReLU'd dots 1, 3, 0, 0.5.  With w = -2 the scores
    are -2, -6, 0, -1, so the largest magnitude belongs to a NEGATIVE score (a max of the signed
    scores would give 0); with w = +2 they are 2, 6, 0, 1."""
    dI, D = 4, 128
    kI = bf16_bits([[1, 0, 0, 0], [3, 0, 0, 0], [-4, 0, 0, 0], [0.5, 0, 0, 0]])
    qI = bf16_bits([[[1, 0, 0, 0]]] * 2)                         # rows t = 0 and t = 3
    rng = np.random.default_rng(9)
    q = rand_bf16(rng, (2, 1, D))
    k = rand_bf16(rng, (4, 1, D))
    v = rand_bf16(rng, (4, 1, D))
    t_rows = np.array([0, 3])
    for wv, absmax, tau, sel in ((-2.0, [2.0, 6.0], [-2.0, -1.0], [2, 3]), (2.0, [2.0, 6.0], [2.0, 2.0], [1, 0])):
        w = bf16_bits([[wv], [wv]])
        r = oracle.dsa_rows(q, qI, w, k, v, kI, t_rows, 2, 1.0, keep_scores=True)
        assert r["absmax"].tolist() == absmax, wv
        assert r["tau"].tolist() == tau, wv
        assert r["idx"][0].tolist() == [0, -1]                  # one causal key at t = 0
        assert r["idx"][1].tolist() == sel, wv
        assert r["scores"][1, :4].tolist() == [wv * 1, wv * 3, 0.0, wv * 0.5]


# ----------------------------------------------------------------------------- top-k


def brute_topk(scores, n, k):
    order = sorted(range(n), key=lambda s: (-scores[s], s))
    sel = order[:min(k, n)]
    return sel + [-1] * (k - len(sel))


def test_topk_brute_force_with_forced_ties():
    """Duplicated kI rows give exactly equal scores; the lower index must win."""
    rng = np.random.default_rng(4)
    L, HI, dI, k = 48, 2, 64, 7
    base = rand_bf16(rng, (6, dI))
    kI = base[rng.integers(0, 6, size=L)]                     # only 6 distinct keys -> many ties
    qI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, HI))
    scores = oracle.index_rows(qI, w, kI, np.arange(L))
    idx, tau = oracle.topk_rows(np.nan_to_num(scores, nan=-np.inf), np.arange(L) + 1, k)
    ties_seen = 0
    for t in range(L):
        want = brute_topk(list(scores[t, :t + 1]), t + 1, k)
        assert list(idx[t]) == want
        row = scores[t, :t + 1]
        if t + 1 > k:
            assert tau[t] == row[want[k - 1]]
            ties_seen += int(np.sum(row == tau[t]) > 1)
    assert ties_seen > 0                                      # the case really exercised ties


def test_topk_tie_rule_on_designed_rows():
    scores = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.0, 3.0]])
    idx, tau = oracle.topk_rows(scores, [7], 3)
    assert list(idx[0]) == [1, 2, 4] and tau[0] == 3.0
    idx, _ = oracle.topk_rows(scores, [7], 5)
    assert list(idx[0]) == [1, 2, 4, 6, 3]
    idx, _ = oracle.topk_rows(np.zeros((1, 9)), [9], 4)      # all equal: first four indices
    assert list(idx[0]) == [0, 1, 2, 3]


def test_topk_invariants_and_short_rows():
    rng = np.random.default_rng(5)
    n_rows, ld, k = 30, 50, 20
    scores = rng.standard_normal((n_rows, ld))
    n_valid = rng.integers(1, ld + 1, size=n_rows)
    idx, _ = oracle.topk_rows(scores, n_valid, k)
    for r in range(n_rows):
        n = n_valid[r]
        sel = idx[r][idx[r] >= 0]
        assert len(sel) == min(k, n) and len(set(sel.tolist())) == len(sel)
        assert np.all(sel < n) and np.all(idx[r][len(sel):] == -1)
        if n <= k:
            assert sorted(sel.tolist()) == list(range(n))     # k >= n: every causal key
        else:
            assert scores[r, sel].min() >= np.sort(scores[r, :n])[::-1][k - 1]


# ----------------------------------------------------------------------------- sparse attention


def dense_causal_sdpa(q, k, v, scale):
    """torch CPU float64 SDPA with GQA heads expanded (contiguous groups)."""
    qt = torch.as_tensor(f64(q)).permute(1, 0, 2)            # [Hq, L, D]
    G = q.shape[1] // k.shape[1]
    kt = torch.as_tensor(f64(k)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.as_tensor(f64(v)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (6, 1)])
def test_sparse_equals_dense_when_k_covers_the_row(Hq, Hkv):
    """k >= L: every causal key is selected, so the result is dense causal attention."""
    rng = np.random.default_rng(6)
    L, D, HI, dI = 33, 16, 2, 8
    q, k, v = rand_bf16(rng, (L, Hq, D)), rand_bf16(rng, (L, Hkv, D)), rand_bf16(rng, (L, Hkv, D))
    qI, kI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, dI)), rand_bf16(rng, (L, HI))
    scale = 1.0 / math.sqrt(D)
    res = oracle.dsa_rows(q, qI, w, k, v, kI, np.arange(L), topk=L + 5, scale=scale)
    np.testing.assert_allclose(res["out"], dense_causal_sdpa(q, k, v, scale), rtol=0, atol=1e-12)


def test_single_selected_key_returns_its_value_row():
    rng = np.random.default_rng(7)
    L, Hq, Hkv, D, HI, dI = 20, 4, 2, 16, 2, 8
    q, k, v = rand_bf16(rng, (L, Hq, D)), rand_bf16(rng, (L, Hkv, D)), rand_bf16(rng, (L, Hkv, D))
    qI, kI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, dI)), rand_bf16(rng, (L, HI))
    res = oracle.dsa_rows(q, qI, w, k, v, kI, np.arange(L), topk=1, scale=0.3, keep_scores=True)
    vf = f64(v)
    for t in range(L):
        row = res["scores"][t, :t + 1]
        s_star = int(np.flatnonzero(row == row.max())[0])
        assert res["idx"][t, 0] == s_star
        for h in range(Hq):
            assert np.array_equal(res["out"][t, h], vf[s_star, h // (Hq // Hkv)])


def test_softmax_normalises_and_constant_values_pass_through():
    """V = 1 everywhere gives exactly 1 (weights sum to 1); identical V rows pass through;
    q = 0 makes every logit equal so lse = log(number of selected keys)."""
    rng = np.random.default_rng(8)
    L, Hq, Hkv, D, HI, dI, topk = 50, 4, 2, 16, 2, 8, 12
    q, k = rand_bf16(rng, (L, Hq, D), 3.0), rand_bf16(rng, (L, Hkv, D), 3.0)
    qI, kI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, dI)), rand_bf16(rng, (L, HI))
    ones = bf16_bits(np.ones((L, Hkv, D)))
    res = oracle.dsa_rows(q, qI, w, k, ones, kI, np.arange(L), topk, 0.2)
    np.testing.assert_allclose(res["out"], 1.0, rtol=0, atol=1e-12)
    row = rand_bf16(rng, (1, Hkv, D))
    same = np.repeat(row, L, axis=0)
    res = oracle.dsa_rows(q, qI, w, k, same, kI, np.arange(L), topk, 0.2)
    G = Hq // Hkv
    for h in range(Hq):
        np.testing.assert_allclose(res["out"][:, h], np.broadcast_to(f64(row)[0, h // G], (L, D)),
                                   rtol=0, atol=1e-12)
    zeros = bf16_bits(np.zeros((L, Hq, D)))
    res = oracle.dsa_rows(zeros, qI, w, k, same, kI, np.arange(L), topk, 0.2)
    n_sel = np.minimum(np.arange(L) + 1, topk)
    np.testing.assert_allclose(res["lse"], np.log(n_sel)[:, None].repeat(Hq, 1), rtol=0, atol=1e-12)


def test_steps_compose_to_the_fused_rows():
    """dsa_rows on a subset of rows equals index_rows -> topk_rows -> sparse_attn_rows."""
    cfg = synth.CONFIGS["tiny"]
    x = synth.inputs(cfg, 0, 300)
    rows = np.array([0, 1, 5, 100, 255, 256, 257, 299])
    res = oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows,
                          cfg.k, cfg.scale, keep_scores=True)
    sc = oracle.index_rows(x["qI"][rows], x["w"][rows], x["kI"], rows)
    np.testing.assert_array_equal(np.nan_to_num(sc, nan=7.0), np.nan_to_num(res["scores"], nan=7.0))
    idx, tau = oracle.topk_rows(np.nan_to_num(sc, nan=-np.inf), rows + 1, cfg.k)
    np.testing.assert_array_equal(idx, res["idx"])
    out, lse = oracle.sparse_attn_rows(x["q"][rows], x["k"], x["v"], idx, cfg.scale)
    np.testing.assert_array_equal(out, res["out"])
    np.testing.assert_array_equal(lse, res["lse"])
    assert np.all(res["idx"][:3, :][res["idx"][:3, :] >= 0] <= 5)


def test_golden_regression_fixture():
    """Stored oracle outputs for a small seeded case (written by tests/golden/make_golden.py,
    which calls only the oracle): guards against accidental changes of the oracle."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_rows.json")
    with open(path) as f:
        g = json.load(f)
    cfg = synth.CONFIGS[g["config"]]
    rows = np.array(g["rows"])
    x = synth.inputs(cfg, 0, int(rows.max()) + 1)
    res = oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows,
                          cfg.k, cfg.scale)
    for r, row in enumerate(g["per_row"]):
        assert sorted(res["idx"][r][res["idx"][r] >= 0].tolist()) == row["idx_sorted"]
        assert res["tau"][r] == pytest.approx(row["tau"], rel=1e-12)
        np.testing.assert_allclose(res["out"][r, :, :4].ravel(), row["out_head_d0_3"], rtol=1e-10, atol=1e-12)


def test_sliding_window_topk_brute_force():
    """SW-DSA: with window W only keys t-W+1..t compete; W >= t+1 is the full causal row and
    W = 1 keeps the query's own key."""
    rng = np.random.default_rng(9)
    L, HI, dI, k = 60, 2, 16, 9
    base = rand_bf16(rng, (5, dI))
    kI = base[rng.integers(0, 5, size=L)]                     # ties again
    qI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, HI))
    scores = oracle.index_rows(qI, w, kI, np.arange(L))
    full = np.nan_to_num(scores, nan=-np.inf)
    for W in (1, 7, 20, 1000):
        idx, _ = oracle.topk_rows(full, np.arange(L) + 1, k, window=W)
        for t in range(L):
            lo = max(0, t - W + 1)
            order = sorted(range(lo, t + 1), key=lambda s: (-scores[t, s], s))[:k]
            assert list(idx[t][:len(order)]) == order and np.all(idx[t][len(order):] == -1)
    idx_w, _ = oracle.topk_rows(full, np.arange(L) + 1, k, window=L + 1)
    idx_f, _ = oracle.topk_rows(full, np.arange(L) + 1, k)
    assert np.array_equal(idx_w, idx_f)
    res = oracle.dsa_rows(rand_bf16(rng, (L, 2, 16)), qI, w, rand_bf16(rng, (L, 1, 16)), rand_bf16(rng, (L, 1, 16)),
                          kI, np.arange(L), k, 0.25, window=1)
    assert np.array_equal(res["idx"][:, 0], np.arange(L)) and np.all(res["idx"][:, 1:] == -1)


# ----------------------------------------------------------------------------- warm-up KL target


def test_kl_two_keys_closed_form():
    """Two keys, one head: logits (0, ln 3) give P = (1/4, 3/4); w = 0 gives uniform Q, so
    KL(P || Q) = ln(27/16) / 4 exactly (the reverse direction would be ln(4/3) / 2)."""
    D, dI = 128, 64
    q = np.zeros((1, 1, D)); q[0, 0, 0] = 1.0
    k = np.zeros((2, 1, D)); k[1, 0, 0] = 1.0
    qI = np.zeros((1, 1, dI)); qI[0, 0, 0] = 1.0
    kI = np.ones((2, dI))
    w = np.zeros((1, 1))
    got = oracle.kl_rows(bf16_bits(q), bf16_bits(k), bf16_bits(qI), bf16_bits(w), bf16_bits(kI), [1], math.log(3.0))
    assert got[0] == pytest.approx(math.log(27.0 / 16.0) / 4.0, rel=1e-13)


def nonneg_bf16(rng, shape):
    x = torch.as_tensor(np.abs(rng.standard_normal(shape)) * 0.3, dtype=torch.float32).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def test_kl_vanishes_when_attention_equals_the_indexer():
    """One head, q = [qI, 0], k = [kI, 0], scale 1, one indexer head of weight 1 and non-negative
    qI, kI (so the ReLU is the identity): the attention logits equal the indexer scores, P = Q
    and KL = 0 on every row, including t = 0."""
    rng = np.random.default_rng(21)
    L, D, dI = 40, 128, 64
    qI = nonneg_bf16(rng, (L, 1, dI))
    kI = nonneg_bf16(rng, (L, dI))
    q = np.zeros((L, 1, D), dtype=np.uint16); q[:, :, :dI] = qI
    k = np.zeros((L, 1, D), dtype=np.uint16); k[:, 0, :dI] = kI
    w = bf16_bits(np.ones((L, 1)))
    rows = np.arange(L)
    got = oracle.kl_rows(q, k, qI, w, kI, rows, 1.0)
    assert np.all(np.abs(got) < 1e-12), got


def test_kl_head_average_and_gibbs():
    """Two query heads with the same query rows give the same P as one head (P is the head
    average, not the sum); KL >= 0 on random rows, = 0 at t = 0 (a single key)."""
    rng = np.random.default_rng(22)
    L, D, HI, dI = 33, 128, 4, 64
    q1 = rand_bf16(rng, (L, 1, D))
    q2 = np.concatenate([q1, q1], axis=1)
    k = rand_bf16(rng, (L, 1, D))
    qI, kI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, dI)), rand_bf16(rng, (L, HI))
    rows = np.arange(L)
    one = oracle.kl_rows(q1, k, qI, w, kI, rows, 0.0883883)
    two = oracle.kl_rows(q2, k, qI, w, kI, rows, 0.0883883)
    np.testing.assert_allclose(two, one, rtol=1e-12, atol=1e-14)
    assert one[0] == pytest.approx(0.0, abs=1e-15)
    assert np.all(one[1:] > 0.0)


def test_kl_gqa_head_map():
    """GQA: with Hq = 4 over Hkv = 2, head h reads KV head h // 2.  Swapping the two KV heads and
    the two query-head pairs together leaves KL unchanged; swapping only the KV heads changes it."""
    rng = np.random.default_rng(23)
    L, D, HI, dI = 20, 128, 2, 64
    q = rand_bf16(rng, (L, 4, D))
    k = rand_bf16(rng, (L, 2, D))
    qI, kI, w = rand_bf16(rng, (L, HI, dI)), rand_bf16(rng, (L, dI)), rand_bf16(rng, (L, HI))
    rows = np.arange(L)
    base = oracle.kl_rows(q, k, qI, w, kI, rows, 0.0883883)
    both = oracle.kl_rows(q[:, [2, 3, 0, 1]], k[:, [1, 0]], qI, w, kI, rows, 0.0883883)
    kv_only = oracle.kl_rows(q, k[:, [1, 0]], qI, w, kI, rows, 0.0883883)
    np.testing.assert_allclose(both, base, rtol=1e-12, atol=1e-14)
    assert np.max(np.abs(kv_only - base)) > 1e-6
