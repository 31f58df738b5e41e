#!/usr/bin/env python
"""Throughput of the DSA hot path on B200: prefill tokens/s at 128K context (headline `value`)
and decode tokens/s for 16 sequences x 128K context, with per-kernel roofline fractions, an
end-to-end number through host buffers, and the fp64 CPU oracle timed on the host cores.

One step = one dsa_prefill over the whole 131072-token sequence (indexer -> top-k -> sparse
attention, all query chunks).  Inputs are seeded synthetic bf16 tensors with the pages' long
video layout (repeating 512 frame tokens + 64 text tokens; block-structured keys), far larger
than L2, resident in HBM when the timed region starts.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun each rank runs its own independent sequence (weak scaling, no collective on the
data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "DSA prefill tokens/s and decode tokens/s @128K ctx, k=2048, 1 B200; % roofline"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------------------------- work accounting
def causal_keys(t0: int, rows: int) -> int:
    """sum_{t=t0}^{t0+rows-1} (t+1)"""
    return rows * t0 + rows * (rows + 1) // 2


def selected_keys(L: int, k: int) -> int:
    """sum_t min(k, t+1)"""
    m = min(L, k)
    return m * (m + 1) // 2 + max(0, L - k) * k


def selected_keys_range(lo: int, hi: int, k: int) -> int:
    """sum_{t=lo}^{hi-1} min(k, t+1)"""
    return selected_keys(hi, k) - selected_keys(lo, k)


def prefill_work(cfg, lo: int = 0, hi: int | None = None) -> dict:
    """Algorithmic work of query rows [lo, hi) of one prefill (default: the whole sequence),
    per kernel kind."""
    hi = cfg.L if hi is None else hi
    n = hi - lo
    caus = causal_keys(lo, n)
    sel = selected_keys_range(lo, hi, cfg.k)
    return {
        "indexer_flop": 2 * cfg.HI * cfg.dI * caus,
        "topk_bytes": 4 * caus + 4 * cfg.k * n,
        "attn_gather_bytes": sel * cfg.Hkv * cfg.D * 2 * 2,
        "attn_io_bytes": n * cfg.Hq * cfg.D * 2 * 2 + 4 * cfg.k * n,
    }


def decode_step_bytes(cfg, ctx_mean: float) -> float:
    """Algorithmic bytes of one decode step for cfg.batch sequences whose keys number ctx_mean on
    average: the kI stream (2*dI bytes per key), the fp32 score row written and read back, the
    K/V gather (k keys x Hkv x D x K and V x 2 bytes) and the idx row written and read back."""
    return cfg.batch * (ctx_mean * cfg.dI * 2 + 2 * 4 * ctx_mean + cfg.k * cfg.Hkv * cfg.D * 2 * 2 + 2 * 4 * cfg.k)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if not self.proc or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle baseline
def cpu_baseline(cfg, x, budget_s: float = 15.0, seed: int = 7) -> dict:
    """The fp64 oracle, as it stands, on a bounded uniform sample of the workload's query rows."""
    import oracle
    cores = oracle.threads()
    # one probe batch to size the sample so the whole leg takes about budget_s
    probe_rows = np.sort(synth.sample_rows(max(2, cores), cfg.L, seed=seed, key=0xC0DE))
    t0 = time.perf_counter()
    oracle.dsa_rows(x["q"][probe_rows], x["qI"][probe_rows], x["w"][probe_rows], x["k"], x["v"], x["kI"], probe_rows,
                    cfg.k, cfg.scale)
    probe = time.perf_counter() - t0
    n = int(max(cores, min(4096, len(probe_rows) * max(1.0, (budget_s - probe) / max(probe, 1e-3)))))
    rows = np.sort(synth.sample_rows(n, cfg.L, seed=seed + 1, key=0xC0DE))
    t0 = time.perf_counter()
    oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows, cfg.k, cfg.scale)
    el = time.perf_counter() - t0
    return {"value": n / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} query rows drawn uniformly from the {cfg.L}-token prefill (full path per row: "
                      f"indexer over t+1 keys, sort-based top-{cfg.k}, attention), {el:.1f} s after a "
                      f"{probe:.1f} s sizing probe of {len(probe_rows)} rows; unbiased for tokens/s since rows "
                      f"are uniform in t"}


# ----------------------------------------------------------------------------- reference arm
def bench_config(cfg, workload: str, world: int, split: str = "seq") -> dict:
    """The `config` object of the JSON line, identical for both arms."""
    if split == "rows":
        par = (f"rows{world} (one sequence; causal-work-balanced query-row ranges per rank, K/V/kI "
               "replicated; output rows assembled on every rank by one broadcast per range)")
    else:
        par = f"dp{world} (independent sequences)"
    return {"workload": f"prefill_{workload}", "L": cfg.L, "k": cfg.k, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D,
            "HI": cfg.HI, "dI": cfg.dI, "batch": 1, "parallelism": par,
            "l2": "inputs (1.8 GB) larger than L2; no flush"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = synth.CONFIGS[args.workload]
    x = synth.inputs(cfg, 0, cfg.L)
    vals = []
    budget = args.ref_seconds if args.ref_seconds else max(5.0, 120.0 / max(1, args.steps + args.warmup))
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(cfg, x, budget_s=budget, seed=11 + i)
        if i >= args.warmup:
            vals.append(cb["value"])
    value = statistics.mean(vals)
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * cfg.L / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(cfg, args.workload, max(1, args.gpus)),
            "cpu_baseline": cb, "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--workload", default="128k", choices=["32k", "128k", "256k"])
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--decode-ctx", type=int, default=0, help="override the cached context (small profiling cases)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="measure only the decode step and print its object (profiling cases)")
    ap.add_argument("--no-kl", action="store_true", help="skip the indexer warm-up KL measurement")
    ap.add_argument("--kl-only", action="store_true",
                    help="measure only the indexer warm-up KL and print its object (profiling cases)")
    ap.add_argument("--kl-rows", type=int, default=0,
                    help="query rows of the 32K workload for the KL measurement (default: all 32768)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-blocks", default="ramp",
                    help="end-to-end leg's row blocks: 'ramp' (small first and last blocks, 16384-row blocks "
                         "between), a size, or 'size x count' items for the first rows then the last size "
                         "repeated (e.g. 8192x8,16384)")
    ap.add_argument("--no-dedup", action="store_true", help="skip the adjacent-query dedup attention measurement")
    ap.add_argument("--dedup-only", action="store_true", help="only the dedup attention measurement (rank 0)")
    ap.add_argument("--dedup-rows", type=int, default=8192, help="query rows of the dedup measurement")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--ref-seconds", type=float, default=0.0,
                    help="oracle seconds per reference-arm step (default: about 2 minutes per run)")
    ap.add_argument("--chunk-rows", type=int, default=0,
                    help="limit the prefill workspace to this many score rows (small profiling cases)")
    ap.add_argument("--split", default="seq", choices=["seq", "rows"],
                    help="under torchrun: seq = one independent sequence per rank (weak scaling); rows = one "
                         "sequence whose query rows are split over the ranks (strong scaling)")
    ap.add_argument("--profile-rows", default="",
                    help="R0:N -- run only query rows R0..R0+N-1 of the workload through dsa_prefill_rows, "
                         "once untimed and once more (a small case for ncu captures); prints its work units")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import dsa_lightning_indexer_02_b200 as dsa
    from dsa_lightning_indexer_02_b200.sharding import (assemble_row_ranges, causal_balanced_row_ranges, reduce_max,
                                                        weak_scaling_value)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dist if world > 1 else None, device="cuda")

    peaks, peak_src = load_peaks()
    if args.kl_only:
        kl = run_kl(torch, dsa, synth.CONFIGS["32k"], barrier, max_over_ranks, peaks, rows=args.kl_rows)
        if rank == 0:
            print(json.dumps({"indexer_kl": kl}), flush=True)
        return 0
    if args.decode_only:
        decode = run_decode(torch, dsa, decode_config(args), args.decode_steps, rank, world, barrier,
                            max_over_ranks, peaks)
        if rank == 0:
            print(json.dumps({"decode": decode}), flush=True)
        return 0
    cfg = synth.CONFIGS[args.workload]
    if args.dedup_only:
        if rank == 0:
            print(json.dumps({"attn_dedup": run_dedup(torch, dsa, cfg, rows=args.dedup_rows)}), flush=True)
        return 0
    if args.profile_rows:
        return run_profile_case(torch, dsa, cfg, args.profile_rows)
    rows_mode = args.split == "rows"
    # split=seq: each rank prefills its own independent sequence (seq = rank); split=rows: every
    # rank holds the same sequence and prefills its causal-work-balanced range of query rows
    x = synth.inputs(cfg, 0, cfg.L, seq=0 if rows_mode else rank)
    ranges = causal_balanced_row_ranges(cfg.L, world, k=cfg.k, align=256 // cfg.HI) if rows_mode else None
    lo, hi = ranges[rank] if rows_mode else (0, cfg.L)
    names = ("q", "k", "v", "qI", "kI", "w")
    host = {n: synth.to_torch(x[n]).pin_memory() for n in names}
    d = {n: host[n].cuda() for n in names}
    out = torch.empty((cfg.L, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((cfg.L, cfg.k), dtype=torch.int32, device="cuda")
    ws_bytes = dsa.workspace_size(dsa.DSA_OP_PREFILL, hi, 1, cfg.Hq, cfg.HI, cfg.k)
    if args.chunk_rows:
        ws_bytes = args.chunk_rows * ((cfg.L + 3) // 4 * 4) * 4 + 4096
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        if rows_mode:
            if hi > lo:
                dsa.dsa_prefill_rows(d["q"][lo:hi], d["k"][:hi], d["v"][:hi], d["qI"][lo:hi], d["kI"][:hi],
                                     d["w"][lo:hi], lo, cfg.k, cfg.scale, out[lo:hi], idx[lo:hi], ws=ws)
            assemble_row_ranges((out, idx), ranges, dist if world > 1 else None)
        else:
            dsa.dsa_prefill(d["q"], d["k"], d["v"], d["qI"], d["kI"], d["w"], cfg.k, cfg.scale, out, idx, ws)

    for _ in range(max(3, args.warmup)):
        step()
    st = dsa.sync_status()
    if st != dsa.DSA_OK:
        raise SystemExit(f"warm-up failed: {dsa.status_string(st)}")

    # ---- timed region: K prefill steps (inputs 1.8 GB, far larger than the 126 MB L2)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        n_launch0 = dsa.launch_count()
        dsa.profile_begin()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    prof = dsa.profile_end()
    launches = dsa.launch_count() - n_launch0
    counters = dsa.read_counters(reset=True)
    if dsa.sync_status() != dsa.DSA_OK:
        raise SystemExit("device error during the timed region")
    ms_step = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
    value = (cfg.L if rows_mode else weak_scaling_value(cfg.L, world, 1.0)) / (ms_step / 1000.0)
    union16 = adjacent_union_stat(idx, cfg, torch)
    clk = clocks.summary()

    # ---- per-kernel roofline (event-timed launches inside the timed region, this rank's rows)
    work = prefill_work(cfg, lo, hi)
    kern = kernel_rooflines(prof, work, args.steps, peaks, args.workload, cfg)
    for kv in kern.values():
        kv["peak_source"] = f"{peak_src}: {kv['peak_source']}"
    dominant = max(kern, key=lambda kk: kern[kk]["ms_per_launch"] * kern[kk]["launches_per_step"])
    kd = kern[dominant]
    roofline = {"bound": kd["bound"], "achieved": kd["achieved"], "peak": kd["peak"], "unit": kd["unit"],
                "frac": kd["frac"], "traffic": kd["traffic"], "kernel": dominant, "peak_source": kd["peak_source"]}
    for extra in ("achieved_logical", "logical_frac", "traffic_scaled_from", "frac_sustained", "note"):
        if extra in kd:
            roofline[extra] = kd[extra]

    # ---- end to end through host buffers and the public row-range call: per block of rows, the
    # host->device copy of its inputs (and of the keys it adds), dsa_prefill_rows, and the
    # device->host copy of its outputs run on three streams, so copies overlap compute
    e2e = None
    if not args.no_e2e:
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hidx = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
        blocks = e2e_blocks(args.e2e_blocks, lo, hi)
        R = max(r1 - r0 for r0, r1 in blocks)
        row_bytes = {n: host[n][0].numel() * host[n].element_size() for n in names}
        # this rank's query rows of q/qI/w, and K/V/kI of every position up to its last row
        h2d = sum(row_bytes[n] * (hi - lo) for n in ("q", "qI", "w")) + \
            sum(row_bytes[n] * hi for n in ("k", "v", "kI"))
        d2h = (hi - lo) * (out[0].numel() * 2 + idx[0].numel() * 4)
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        # score rows of one block at the longest row length, plus alignment slack
        ws_rows = torch.empty(R * ((cfg.L + 3) // 4 * 4) * 4 + 4096, dtype=torch.uint8, device="cuda")

        def e2e_step():
            ev_in = [torch.cuda.Event() for _ in blocks]
            ev_c = [torch.cuda.Event() for _ in blocks]
            s_in.wait_stream(stream)
            if lo > 0:                       # the key prefix that rows before this rank's range hold
                with torch.cuda.stream(s_in):
                    for n in ("k", "v", "kI"):
                        d[n][:lo].copy_(host[n][:lo], non_blocking=True)
            for i, (r0, r1) in enumerate(blocks):
                with torch.cuda.stream(s_in):
                    for n in names:
                        d[n][r0:r1].copy_(host[n][r0:r1], non_blocking=True)
                    ev_in[i].record(s_in)
                s_cmp.wait_event(ev_in[i])
                with torch.cuda.stream(s_cmp):
                    dsa.dsa_prefill_rows(d["q"][r0:r1], d["k"][:r1], d["v"][:r1], d["qI"][r0:r1], d["kI"][:r1],
                                         d["w"][r0:r1], r0, cfg.k, cfg.scale, out[r0:r1], idx[r0:r1], ws=ws_rows,
                                         stream=s_cmp)
                    ev_c[i].record(s_cmp)
                s_out.wait_event(ev_c[i])
                with torch.cuda.stream(s_out):
                    hout[r0:r1].copy_(out[r0:r1], non_blocking=True)
                    hidx[r0:r1].copy_(idx[r0:r1], non_blocking=True)
            stream.wait_stream(s_out)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        ev1.record(stream)
        torch.cuda.synchronize()
        if dsa.sync_status() != dsa.DSA_OK:
            raise SystemExit("device error in the end-to-end leg")
        ms_e2e = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
        e2e = {"value": (cfg.L if rows_mode else weak_scaling_value(cfg.L, world, 1.0)) / (ms_e2e / 1e3),
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "how": f"dsa_prefill_rows over {len(blocks)} blocks of up to {R} rows ({args.e2e_blocks}); H2D, "
                      "compute and D2H on "
                      "three streams, pinned host buffers" +
                      ("; each rank copies in its own query rows and the key prefix they need, and copies "
                       "out its own output rows" if rows_mode else "")}

    del d, host, out, idx, ws
    torch.cuda.empty_cache()

    # ---- decode: 16 sequences x 131072 cached tokens, 256 steps
    decode = None
    if not args.no_decode:
        decode = run_decode(torch, dsa, decode_config(args), args.decode_steps, rank, world, barrier,
                            max_over_ranks, peaks)

    # ---- indexer warm-up KL target on the 32K workload (dense, tensor-core bound)
    kl = None
    if not args.no_kl:
        kl = run_kl(torch, dsa, synth.CONFIGS["32k"], barrier, max_over_ranks, peaks, rows=args.kl_rows)

    # ---- adjacent-query dedup attention against the per-token kernel (last 8192 rows)
    dedup = None
    if not args.no_dedup and rank == 0 and world == 1:
        dedup = run_dedup(torch, dsa, cfg, rows=args.dedup_rows)

    cpu = None
    if rank == 0 and not args.no_cpu and world == 1:
        cpu = cpu_baseline(cfg, x, budget_s=args.cpu_seconds)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if rows_mode else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; 512 frame + 64 text token layout, block-structured keys)",
            "config": bench_config(cfg, args.workload, world, args.split),
            "roofline": roofline, "kernels": kern, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk, "decode": decode, "indexer_kl": kl, "adjacent_union_16": union16, "attn_dedup": dedup,
            "path_counters": counters}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def adjacent_union_stat(idx, cfg, torch, windows: int = 32) -> dict:
    """Mean size of the union of 16 adjacent index sets (rows t..t+15, t >= k) on evenly spaced
    windows: the statistic the pages quote for their adjacent-query dedup (about 8000 of 32768
    at 128K, k = 2048)."""
    starts = np.linspace(cfg.k, cfg.L - 16, windows).astype(np.int64)
    sizes = []
    for t0 in starts:
        rows = idx[int(t0):int(t0) + 16].cpu().numpy()
        sizes.append(len(np.unique(rows[rows >= 0])))
    return {"mean_unique": float(np.mean(sizes)), "naive": 16 * cfg.k, "windows": windows}


def run_dedup(torch, dsa, cfg, rows: int = 8192, reps: int = 3) -> dict:
    """dsa_sparse_attn_dedup against dsa_sparse_attn on the workload's last `rows` query rows:
    (a) with their own top-k index sets, (b) with index sets that have the pages' adjacent-query
    overlap (each block of 16 adjacent rows draws its rows' 2048 keys from one pool of 8000 keys,
    about 7900 distinct per block; rows in the top-k's region order).  Per case: ms per launch of
    each kernel (CUDA events, median of `reps` after one untimed call), the mean number of distinct
    keys per 16 adjacent rows, and the largest output difference between the two kernels."""
    L, C = cfg.L, rows
    t0 = L - C
    d = {n: synth.to_torch(synth.tensor(cfg, n, 0, L)).cuda() for n in ("k", "v", "kI")}
    r = {n: synth.to_torch(synth.tensor(cfg, n, t0, C)).cuda() for n in ("q", "qI", "w")}
    o1 = torch.empty((C, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    own = torch.empty((C, cfg.k), dtype=torch.int32, device="cuda")
    dsa.dsa_prefill_rows(r["q"], d["k"], d["v"], r["qI"], d["kI"], r["w"], t0, cfg.k, cfg.scale, o1, own)
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    nb, pool = C // 16, 8000
    pools = torch.argsort(torch.rand(nb, t0, device="cuda", generator=g), dim=1)[:, :pool]
    pick = torch.argsort(torch.rand(C, pool, device="cuda", generator=g), dim=1)[:, :cfg.k]
    ov = torch.gather(pools.repeat_interleave(16, dim=0), 1, pick).to(torch.int32)
    region_key = ((ov // 32) % 4).to(torch.int64) * (1 << 40) + ov.to(torch.int64)
    ov = torch.gather(ov, 1, torch.argsort(region_key, dim=1)).contiguous()
    del pools, pick, region_key

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        if dsa.sync_status() != dsa.DSA_OK:
            raise SystemExit("device error in the dedup measurement")
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.median(ts))

    res = {"rows": [t0, L]}
    for name, ii in (("own_topk", own), ("pages_overlap", ov)):
        ms_t = timed(lambda: dsa.dsa_sparse_attn(r["q"], d["k"], d["v"], ii, t0, cfg.scale, o1))
        ms_d = timed(lambda: dsa.dsa_sparse_attn_dedup(r["q"], d["k"], d["v"], ii, t0, cfg.scale, o2))
        blocks = ii[: 16 * 64].cpu().numpy().reshape(64, 16 * cfg.k)
        res[name] = {"per_token_ms": round(ms_t, 4), "dedup_ms": round(ms_d, 4),
                     "union16_mean": float(np.mean([len(np.unique(b[b >= 0])) for b in blocks])),
                     "max_abs_diff": float((o1.float() - o2.float()).abs().max())}
    del d, r, o1, o2, own, ov
    torch.cuda.empty_cache()
    return res


# the prefill kernels' algorithmic unit (the denominator of the DRAM bytes per unit in
# profiles/traffic.json): indexer causal score pairs, top-k algorithmic bytes, logical gathered bytes
TRAFFIC_UNITS = {"indexer": "causal (t, s) score pairs", "topk": "algorithmic bytes",
                 "sparse_attn": "logical gathered K/V bytes"}


def traffic_units(cfg, work: dict) -> dict:
    return {"indexer": work["indexer_flop"] / (2 * cfg.HI * cfg.dI), "topk": work["topk_bytes"],
            "sparse_attn": work["attn_gather_bytes"]}


# The gather ceiling of the attention kernel's copy structure when the rows are L2-resident: the same
# ring of bulk copies (3 producer warps, 2 CTAs per SM) with consumers that only release the slots,
# measured on one B200 at 1965 MHz (about 17 TB/s of 1 KiB rows; plain 16-byte loads of L2-resident
# rows reach about 21 TB/s).  Most of the attention's gathered rows hit L2, so this, not the HBM
# copy rate, is the ceiling its logical gather rate is compared with.
L2_GATHER_GBS = 17000.0
L2_GATHER_SOURCE = "bulk-copy ring with trivial consumers, L2-resident 1 KiB rows, one B200 (probe)"


def kernel_rooflines(prof: dict, work: dict, steps: int, peaks: dict, workload: str, cfg) -> dict:
    """Per prefill kernel: mean CUDA-event launch time inside the timed region, achieved rate of
    its algorithmic work, and the fraction of the measured peak for its bound.  The indexer is
    compared with the burst bf16 GEMM rate (it runs at the maximum SM clock inside the step; the
    sustained figure is given alongside).  Sparse attention's roofline is HBM: its fraction is the
    DRAM bytes one launch really moves (ncu, small case scaled per logical gathered byte) over its
    time; the logical gather rate, which L2 reuse lifts past the HBM copy rate, is reported
    separately as achieved_logical / logical_frac."""
    hbm = peaks["hbm_gbs"]
    burst = peaks["bf16_tflops"]
    sust = peaks.get("bf16_tflops_sustained", burst)
    kern = {}

    def per_launch(kind):
        p = prof[kind]
        return p["ms"] / max(1, p["launches"]), p["launches"] / steps

    ms_i, n_i = per_launch("indexer")
    ms_t, n_t = per_launch("topk")
    ms_a, n_a = per_launch("sparse_attn")
    # algorithmic units per launch = per-step work / launches per step (the step totals are exact;
    # per-launch figures are their mean over the chunks)
    ach_i = work["indexer_flop"] / n_i / (ms_i / 1e3) / 1e12
    kern["indexer"] = {"bound": "tensor", "achieved": ach_i, "peak": burst, "unit": "TFLOP/s", "frac": ach_i / burst,
                       "frac_sustained": ach_i / sust, "ms_per_launch": ms_i, "launches_per_step": n_i,
                       "peak_source": "measured burst bf16 (MEASURED_PEAKS.json bf16_tflops); sustained alongside"}
    ach_t = work["topk_bytes"] / n_t / (ms_t / 1e3) / 1e9
    kern["topk"] = {"bound": "hbm", "achieved": ach_t, "peak": hbm, "unit": "GB/s", "frac": ach_t / hbm,
                    "ms_per_launch": ms_t, "launches_per_step": n_t, "peak_source": "measured HBM copy"}
    logical = (work["attn_gather_bytes"] + work["attn_io_bytes"]) / n_a / (ms_a / 1e3) / 1e9
    kern["sparse_attn"] = {"bound": "hbm", "achieved": logical, "peak": hbm, "unit": "GB/s", "frac": logical / hbm,
                           "achieved_logical": logical, "logical_frac": logical / hbm, "ms_per_launch": ms_a,
                           "launches_per_step": n_a, "peak_source": "measured HBM copy",
                           "l2_gather_ceiling": {"value": L2_GATHER_GBS, "unit": "GB/s", "frac": logical / L2_GATHER_GBS,
                                                 "source": L2_GATHER_SOURCE}}
    # DRAM bytes per launch: ncu counters of a small case of the same kernel, scaled by the
    # launch's algorithmic units, used only while the kernel code (comments aside) is unchanged
    tr = {}
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tr = json.load(f)
    sha = lib_hash()
    units = traffic_units(cfg, work)
    n_per = {"indexer": n_i, "topk": n_t, "sparse_attn": n_a}
    for name, kd in kern.items():
        ent = tr.get(name)
        kd["traffic"] = None
        if ent and ent.get("lib_sha") == sha and ent.get("workload") == workload:
            kd["traffic"] = ent["bytes_per_unit"] * units[name] / n_per[name]
            kd["traffic_scaled_from"] = ent["case"]
            kd["dram_gbs"] = kd["traffic"] / (kd["ms_per_launch"] / 1e3) / 1e9
    ka = kern["sparse_attn"]
    if ka["traffic"] is not None:
        ka["achieved"] = ka["dram_gbs"]
        ka["frac"] = ka["dram_gbs"] / hbm
        ka["note"] = ("achieved/frac: DRAM bytes moved per launch over its time; most gathered rows hit L2, "
                      "so the logical gather rate (achieved_logical) exceeds the HBM copy rate")
    else:
        ka["note"] = ("no DRAM capture for these sources: achieved/frac fall back to the logical gather rate, "
                      "which L2 reuse lifts past the HBM copy rate")
    return kern


def run_profile_case(torch, dsa, cfg, spec: str) -> int:
    """Query rows R0..R0+N-1 of the workload through dsa_prefill_rows with a workspace that holds
    all N score rows (one launch of each kernel per call), once untimed and once more.  The small
    case that ncu captures: a few GB on the device, one launch per kernel per call."""
    r0, n = (int(v) for v in spec.split(":"))
    hi = r0 + n
    assert 0 <= r0 and n > 0 and hi <= cfg.L
    d = {}
    for name in ("k", "v", "kI"):
        d[name] = synth.to_torch(synth.tensor(cfg, name, 0, hi)).cuda()
    for name in ("q", "qI", "w"):
        d[name] = synth.to_torch(synth.tensor(cfg, name, r0, n)).cuda()
    out = torch.empty((n, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((n, cfg.k), dtype=torch.int32, device="cuda")
    ws = torch.empty(n * ((hi + 3) // 4 * 4) * 4 + 4096, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        dsa.dsa_prefill_rows(d["q"], d["k"], d["v"], d["qI"], d["kI"], d["w"], r0, cfg.k, cfg.scale, out, idx, ws=ws)
    torch.cuda.synchronize()
    if dsa.sync_status() != dsa.DSA_OK:
        raise SystemExit("device error in the profiling case")
    work = prefill_work(cfg, r0, hi)
    print(json.dumps({"profile_rows": [r0, n], "workload": cfg.name, "lib_sha": lib_hash(),
                      "units_per_launch": traffic_units(cfg, work), "unit_names": TRAFFIC_UNITS}), flush=True)
    return 0


E2E_RAMP_HEAD = (2048, 2048, 4096, 4096, 8192, 8192)
E2E_RAMP_TAIL = (8192, 4096)


def e2e_blocks(spec: str, lo: int, hi: int) -> list:
    """Row blocks [r0, r1) covering [lo, hi) for the end-to-end leg.  spec 'ramp': small blocks
    first (their host-to-device copies are what the first compute waits for) and last (their
    device-to-host copies are what the step waits for after the last compute), 16384-row blocks
    between (longer launches run faster); a range too short for that takes 8192-row blocks.  Else
    comma-separated items 'size' or 'size x count', used in order, the last size repeating.
    Measured at 128K: uniform 8192-row blocks 1.306 M tokens/s, the ramp 1.322 M."""
    if spec == "ramp":
        n = hi - lo
        fixed = sum(E2E_RAMP_HEAD) + sum(E2E_RAMP_TAIL)
        if n <= fixed:
            return [(r, min(hi, r + 8192)) for r in range(lo, hi, 8192)]
        mid = n - fixed
        sizes = list(E2E_RAMP_HEAD) + [16384] * (mid // 16384) + ([mid % 16384] if mid % 16384 else []) + \
            list(E2E_RAMP_TAIL)
        blocks, r = [], lo
        for sz in sizes:
            blocks.append((r, r + sz))
            r += sz
        return blocks
    items = []
    for it in spec.split(","):
        size, _, count = it.strip().partition("x")
        items.append((int(size), int(count) if count else None))
    blocks, r, i = [], lo, 0
    while r < hi:
        size, count = items[min(i, len(items) - 1)]
        n = count if (count and i < len(items)) else 1
        for _ in range(n):
            if r >= hi:
                break
            blocks.append((r, min(hi, r + size)))
            r = blocks[-1][1]
        i += 1
    return blocks


def source_code_only(text: str) -> str:
    """Kernel source without comments and blank lines (no string literal in csrc/ holds '//'
    or '/*'), so that a comment edit does not mark the ncu counters of unchanged code stale."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def lib_hash() -> str:
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "dsa_lightning_indexer_02_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(source_code_only(f.read()).encode())
    return h.hexdigest()[:12]


def run_kl(torch, dsa, cfg, barrier, max_over_ranks, peaks, reps: int = 3, rows: int = 0):
    """dsa_indexer_kl over one sequence of the workload (its first `rows` tokens, default all):
    KL(P_t || Q_t) for every query row (indexer scores per chunk, then the dense two-pass
    kernel); tokens/s and the dense kernel's fraction of the bf16 tensor peak (4 x Hq x D flop
    per causal pair).  One untimed call, then `reps` timed calls."""
    L = min(rows, cfg.L) if rows > 0 else cfg.L
    x = {n: synth.to_torch(synth.tensor(cfg, n, 0, L)).cuda() for n in ("q", "k", "qI", "kI", "w")}
    kl = torch.empty(L, dtype=torch.float32, device="cuda")
    ws = torch.empty(dsa.workspace_size(dsa.DSA_OP_INDEXER_KL, L, 1, cfg.Hq, cfg.HI, 1), dtype=torch.uint8,
                     device="cuda")

    def run():
        dsa.dsa_indexer_kl(x["q"], x["k"], x["qI"], x["kI"], x["w"], cfg.scale, kl, ws)

    run()
    torch.cuda.synchronize()
    if dsa.sync_status() != dsa.DSA_OK:
        raise SystemExit("indexer KL warm-up failed")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    dsa.profile_begin()
    ev0.record()
    for _ in range(reps):
        run()
    ev1.record()
    torch.cuda.synchronize()
    prof = dsa.profile_end()
    ms = max_over_ranks(ev0.elapsed_time(ev1)) / reps
    pairs = L * (L + 1) / 2
    flop = 4.0 * cfg.Hq * cfg.D * pairs
    k_ms = prof["kl"]["ms"] / reps
    achieved = flop / (k_ms / 1e3) / 1e12
    tpeak = peaks["bf16_tflops"]                     # the kernel is timed on its own: burst peak
    tsust = peaks.get("bf16_tflops_sustained", tpeak)
    return {"workload": "prefill_32k" if L == cfg.L else f"prefill_32k_first_{L}", "value": L / (ms / 1e3),
            "unit": "tokens/s", "ms_per_sequence": ms,
            "kernel_ms": k_ms, "indexer_ms": prof["indexer"]["ms"] / reps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tpeak,
                         "unit": "TFLOP/s", "frac": achieved / tpeak, "frac_sustained": achieved / tsust,
                         "algorithmic": "4 x Hq x D flop per causal (t, s) pair (two passes of Q.K)"},
            "mean_kl": float(kl.mean()), "mma": "tcgen05 (TMEM accumulators, TMA operands)"}


def decode_config(args):
    """The decode workload (16 sequences x 131072 cached tokens), or a shorter cached context."""
    dcfg = synth.CONFIGS["decode"]
    if args.decode_ctx:
        import dataclasses
        dcfg = dataclasses.replace(dcfg, L=args.decode_ctx, iid_from=args.decode_ctx)
    return dcfg


def run_decode(torch, dsa, cfg, steps, rank, world, barrier, max_over_ranks, peaks):
    B, ctx0 = cfg.batch, cfg.L
    Lmax = ctx0 + steps
    kc = torch.empty((B, Lmax, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    kIc = torch.empty((B, Lmax, cfg.dI), dtype=torch.bfloat16, device="cuda")
    newt = {n: [] for n in ("q", "qI", "w", "k", "v", "kI")}
    for b in range(B):
        seq = rank * B + b
        for n, dst in (("k", kc), ("v", vc), ("kI", kIc)):
            dst[b, :ctx0].copy_(synth.to_torch(synth.tensor(cfg, n, 0, ctx0, seq=seq)))
        for n in newt:
            newt[n].append(synth.to_torch(synth.tensor(cfg, n, ctx0, steps, seq=seq)))
    # per step j: tensors [B, ...] of token ctx0 + j
    new = {n: torch.stack(newt[n], dim=1).cuda().contiguous() for n in newt}
    ctx = torch.full((B,), ctx0, dtype=torch.int32, device="cuda")
    out = torch.empty((B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dsa.workspace_size(dsa.DSA_OP_DECODE, Lmax, B, cfg.Hq, cfg.HI, cfg.k), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.current_stream()

    def one(j):
        dsa.dsa_decode(new["q"][j], new["qI"][j], new["w"][j], new["k"][j], new["v"][j], new["kI"][j], kc, vc,
                       kIc, ctx, cfg.k, cfg.scale, out, ws=ws, update_ctx=True)

    for j in range(min(8, steps)):
        one(j)
    torch.cuda.synchronize()
    ctx.fill_(ctx0)
    if dsa.sync_status() != dsa.DSA_OK:
        raise SystemExit("decode warm-up failed")
    # the whole loop of `steps` decode steps as one CUDA graph (ctx_len advances on the device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for j in range(steps):
            one(j)
    torch.cuda.synchronize()
    ctx.fill_(ctx0)
    graph.replay()                       # warm replay
    torch.cuda.synchronize()
    ctx.fill_(ctx0)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    if dsa.sync_status() != dsa.DSA_OK or int(ctx[0]) != ctx0 + steps:
        raise SystemExit("decode graph replay failed")
    ms = max_over_ranks(ev0.elapsed_time(ev1))
    del graph
    # per-kernel breakdown: a separate eager pass with CUDA events around every launch
    ctx.fill_(ctx0)
    torch.cuda.synchronize()
    dsa.profile_begin()
    for j in range(steps):
        one(j)
    torch.cuda.synchronize()
    prof = dsa.profile_end()
    dcount = dsa.read_counters(reset=True)
    kmeans = {k: v["ms"] / steps for k, v in prof.items() if v["launches"]}
    bytes_step = decode_step_bytes(cfg, ctx0 + (steps - 1) / 2)
    return {"value": world * B * steps / (ms / 1e3), "unit": UNIT, "steps": steps, "batch": B, "ctx": ctx0,
            "ms_per_decode_step": ms / steps, "timing": "one CUDA graph of all steps, CUDA events around it",
            "kernel_ms_per_step": kmeans,
            "hbm_frac": bytes_step / (ms / steps / 1e3) / 1e9 / peaks["hbm_gbs"],
            "algorithmic_bytes_per_step": bytes_step, "path_counters": dcount}


if __name__ == "__main__":
    sys.exit(main())
