"""Writes oracle_tiny_rows.json: oracle outputs for a few rows of the seeded 'tiny' workload.

Calls only the oracle and the input generator.  The stored values guard the oracle against
accidental change; they are not a source of truth about the method (the pins in
tests/test_oracle_pins.py are).
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    cfg = synth.CONFIGS["tiny"]
    rows = np.array([0, 7, 255, 256, 511, 1023])
    x = synth.inputs(cfg, 0, int(rows.max()) + 1)
    res = oracle.dsa_rows(x["q"][rows], x["qI"][rows], x["w"][rows], x["k"], x["v"], x["kI"], rows,
                          cfg.k, cfg.scale)
    per_row = []
    for r in range(len(rows)):
        idx = res["idx"][r]
        per_row.append({"t": int(rows[r]),
                        "idx_sorted": sorted(idx[idx >= 0].tolist()),
                        "tau": float(res["tau"][r]),
                        "out_head_d0_3": res["out"][r, :, :4].ravel().tolist()})
    with open(os.path.join(HERE, "oracle_tiny_rows.json"), "w") as f:
        json.dump({"config": "tiny", "rows": rows.tolist(), "per_row": per_row}, f)


if __name__ == "__main__":
    main()
