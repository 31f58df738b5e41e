"""The algorithmic work that bench.py divides by measured time to get each kernel's roofline
fraction: checked against brute force on small cases and against figures derived by hand from
the workload shapes (indexer 2*HI*dI flop per causal pair, top-k 4 bytes per causal score plus
4 per index, gather 2 KiB per selected key at 4 KV heads x 128, decode kI stream + scores +
gather + idx)."""
import pytest

import bench
import synth


@pytest.mark.parametrize("t0,rows", [(0, 1), (0, 17), (5, 9), (1000, 37)])
def test_causal_keys_is_the_sum_of_row_lengths(t0, rows):
    assert bench.causal_keys(t0, rows) == sum(t + 1 for t in range(t0, t0 + rows))


def test_causal_keys_add_up_over_chunks():
    L, C = 131072, 8192
    assert sum(bench.causal_keys(t0, min(C, L - t0)) for t0 in range(0, L, C)) == L * (L + 1) // 2


@pytest.mark.parametrize("L,k", [(1, 1), (5, 8), (8, 8), (9, 8), (300, 16), (1024, 256)])
def test_selected_keys_is_the_sum_of_selection_sizes(L, k):
    assert bench.selected_keys(L, k) == sum(min(k, t + 1) for t in range(L))


# (workload, indexer flop, top-k bytes, logical gather bytes), each to 3 significant digits
_FIGURES = [
    ("32k", 2.20e12, 2.42e9, 1.33e11),
    ("128k", 3.52e13, 3.54e10, 5.45e11),
    ("256k", 1.41e14, 1.40e11, 1.10e12),
]


@pytest.mark.parametrize("name,flop,topk_bytes,gather_bytes", _FIGURES)
def test_prefill_work_matches_hand_figures(name, flop, topk_bytes, gather_bytes):
    w = bench.prefill_work(synth.CONFIGS[name])
    assert w["indexer_flop"] == pytest.approx(flop, rel=5e-3)
    assert w["topk_bytes"] == pytest.approx(topk_bytes, rel=5e-3)
    assert w["attn_gather_bytes"] == pytest.approx(gather_bytes, rel=5e-3)


def test_prefill_work_exact_at_128k():
    c = synth.CONFIGS["128k"]
    L, k = 131072, 2048
    causal = L * (L + 1) // 2
    sel = k * (k + 1) // 2 + (L - k) * k
    w = bench.prefill_work(c)
    assert w["indexer_flop"] == 2 * 32 * 64 * causal
    assert w["topk_bytes"] == 4 * causal + 4 * k * L
    assert w["attn_gather_bytes"] == sel * 2048          # K and V rows of 4 KV heads x 128 bf16
    assert w["attn_io_bytes"] == L * 32 * 128 * 2 * 2 + 4 * k * L


def test_decode_step_bytes_at_16x128k():
    c = synth.CONFIGS["decode"]
    ctx = 131072 + 127.5                                  # mean cached keys over 256 steps
    per_seq = ctx * 128 + 8 * ctx + 2048 * 2048 + 8 * 2048
    assert bench.decode_step_bytes(c, ctx) == pytest.approx(16 * per_seq)
    assert bench.decode_step_bytes(c, ctx) == pytest.approx(3.53e8, rel=5e-3)


def test_source_hash_ignores_comments_only():
    """profiles/traffic.json's counters are keyed by bench.lib_hash(): comment and blank-line edits
    keep the key, any code edit changes it."""
    code = "__global__ void k(int* p) {\n    p[0] = 1;  // store\n}\n"
    commented = "// a kernel\n\n/* block\n   comment */\n__global__ void k(int* p) {\n    p[0] = 1;\n}\n"
    changed = "__global__ void k(int* p) {\n    p[0] = 2;  // store\n}\n"
    assert bench.source_code_only(code) == bench.source_code_only(commented)
    assert bench.source_code_only(code) != bench.source_code_only(changed)


def test_committed_traffic_matches_the_sources():
    """The committed DRAM counters were taken on the kernel code now in csrc/ (else the bench would
    report traffic null)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles",
                           "traffic.json")) as f:
        t = json.load(f)
    for name in ("indexer", "topk", "sparse_attn"):
        assert t[name]["lib_sha"] == bench.lib_hash(), name


@pytest.mark.parametrize("spec", ["ramp", "8192", "8192x8,16384", "4096x4,8192x4,16384x4,8192"])
@pytest.mark.parametrize("lo,hi", [(0, 131072), (0, 262144), (0, 32768), (0, 1000), (65536, 131072), (5, 50000)])
def test_e2e_blocks_partition_the_rows(spec, lo, hi):
    """The end-to-end leg's blocks cover [lo, hi) exactly, in order, without gaps or overlap, so its
    copies and timing count every row once."""
    b = bench.e2e_blocks(spec, lo, hi)
    assert b[0][0] == lo and b[-1][1] == hi
    assert all(b[i][1] == b[i + 1][0] for i in range(len(b) - 1))
    assert all(r1 > r0 for r0, r1 in b)
