"""Write tests/golden/tiny_oracle_rows.json from the float64 oracle only.

The SANA-Video pages print no input/output values for the attention op, so
the only stored expected values are the oracle's own, recorded once so that a
later edit of the oracle's arithmetic shows up as a diff.  Inputs come from the
seeded generator (tiny config: B1 H2 d32 fp32, 12x4x4 latent, blocks of 3
frames, RoPE split (8,12,12), theta 1e4, eps 1e-6).

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

ROWS = [0, 1, 47, 48, 95, 96, 143, 144, 191]


def main():
    w = workloads.CONFIGS["tiny"]
    q, k, v = workloads.call_tensors(w)
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    out = oracle.attention_rows(q, k, v, pos, blk, ROWS, w.split, w.theta, w.eps)
    doc = {
        "what": "float64 oracle outputs o[h][row][:] for the tiny workload, seed 0",
        "workload": {"B": w.B, "H": w.H, "d": w.d, "T": w.T, "Hg": w.Hg, "Wg": w.Wg, "F": w.F,
                     "split": list(w.split), "theta": w.theta, "eps": w.eps, "seed": w.seed},
        "rows": ROWS,
        "out": [[[float(x).hex() for x in out[h, i]] for i in range(len(ROWS))] for h in range(w.H)],
    }
    with open(os.path.join(os.path.dirname(__file__), "tiny_oracle_rows.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
