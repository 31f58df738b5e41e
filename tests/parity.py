"""Comparison rules between the CUDA path and the fp64 oracle.

Index sets: equal per row, except keys whose ORACLE score lies in the near-tie band around the
oracle's k-th score tau:  |score - tau| <= 1e-3 * |tau| + 1e-6 * max_s |score(t, s)|.  The
absolute floor covers rows whose k-th score is exactly 0 or tiny (sign flips of fp32 noise near
zero); exact ties are still decided by the index rule on both sides.

Attention output (bf16 in, fp32 accumulate): max-abs <= 2e-2 and mean-abs <= 2e-3 against the
oracle evaluated on the GPU's own index set.
"""
from __future__ import annotations

import numpy as np

BAND_REL = 1e-3
BAND_ABS_OF_MAX = 1e-6
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3


def index_set_mismatch(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, tau: np.ndarray,
                       absmax: np.ndarray, n_valid: np.ndarray) -> dict:
    """Compare per-row index sets.  ora_scores[r] holds the oracle score row (index = key).

    Returns counts of rows with any difference, keys outside the band, and structural errors.
    """
    rows_diff = keys_diff = out_of_band = structural = 0
    for r in range(gpu_idx.shape[0]):
        n = int(n_valid[r])
        m = min(gpu_idx.shape[1], n)
        g = gpu_idx[r]
        gs = g[g >= 0]
        if len(gs) != m or np.any(g[m:] != -1) or len(np.unique(gs)) != m or np.any(gs >= n):
            structural += 1
            continue
        o = ora_idx[r][ora_idx[r] >= 0]
        sym = np.setxor1d(gs, o)
        if len(sym):
            rows_diff += 1
            keys_diff += len(sym)
            band = BAND_REL * abs(tau[r]) + BAND_ABS_OF_MAX * absmax[r]
            out_of_band += int(np.sum(np.abs(ora_scores[r, sym] - tau[r]) > band))
    return {"rows_diff": rows_diff, "keys_diff": keys_diff, "out_of_band": out_of_band, "structural": structural}


def output_error(gpu_out: np.ndarray, ref_out: np.ndarray) -> dict:
    err = np.abs(gpu_out.astype(np.float64) - ref_out)
    return {"max_abs": float(err.max()) if err.size else 0.0, "mean_abs": float(err.mean()) if err.size else 0.0}


def assert_output_ok(gpu_out, ref_out, what=""):
    e = output_error(gpu_out, ref_out)
    assert e["max_abs"] <= OUT_MAX_ABS and e["mean_abs"] <= OUT_MEAN_ABS, f"{what} {e}"
    return e


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()
