"""The seeded input generator: determinism, slicing, distributions and token layouts."""
import json
import os

import numpy as np
import torch

import synth


def test_deterministic_and_slice_independent():
    cfg = synth.CONFIGS["32k"]
    a = synth.tensor(cfg, "kI", 0, 600)
    b = synth.tensor(cfg, "kI", 0, 600)
    c = synth.tensor(cfg, "kI", 250, 100)
    assert np.array_equal(a, b) and np.array_equal(a[250:350], c)
    assert not np.array_equal(synth.tensor(cfg, "q", 0, 4, seq=0), synth.tensor(cfg, "q", 0, 4, seq=1))


def test_iid_moments_and_bf16_rounding():
    cfg = synth.CONFIGS["tiny"]
    x = synth.bf16_to_f64(synth.tensor(cfg, "q", 0, 1024))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # every value is a bf16 value and survives a bf16 round trip unchanged
    t = torch.as_tensor(x.ravel()[:10000], dtype=torch.float32)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float32), t)


def test_block_structure_of_keys():
    cfg = synth.CONFIGS["128k"]
    ids = synth.block_ids(cfg, 0, 1200)
    assert ids[0] == 0 and ids[511] == 0 and ids[512] == -1 and ids[575] == -1 and ids[576] == 1
    kI = synth.bf16_to_f64(synth.tensor(cfg, "kI", 0, 1200))
    frame0 = kI[:512]
    # frame tokens = mean + 0.5 noise: per-channel spread inside a frame is ~0.5
    assert abs(frame0.std(axis=0).mean() - 0.5) < 0.05
    text = kI[512:576]
    assert abs(text.std() - 1.0) < 0.1
    q = synth.bf16_to_f64(synth.tensor(cfg, "q", 0, 512))
    assert abs(q.std(axis=0).mean() - 1.0) < 0.05          # queries are not block-structured


def test_layouts_of_all_workloads():
    c5 = synth.CONFIGS["256k"]
    ids = synth.block_ids(c5, 0, 600)
    assert (ids[:16] == -1).all() and (ids[16:256] == 0).all() and (ids[256:272] == -1).all()
    c4 = synth.CONFIGS["decode"]
    ids = synth.block_ids(c4, 131000, 328)
    assert (ids[72:] == -1).all()                          # new decode tokens are iid text
    c2 = synth.CONFIGS["32k"]
    assert synth.block_ids(c2, 0, 32768).max() == 127


def test_workloads_follow_the_pages_facts():
    with open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")) as f:
        facts = json.load(f)
    for name in ("32k", "128k", "decode", "256k"):
        assert synth.CONFIGS[name].k == facts["top_k"]["value"]
    assert synth.CONFIGS["128k"].L == facts["measure_context"]["value"]
    assert synth.CONFIGS["decode"].L == facts["measure_context"]["value"]
    assert synth.CONFIGS["256k"].L == facts["max_context"]["value"]
