"""Write tests/golden/tiny_f32_oracle.json from the CPU oracle (and the seeded inputs) only.

The fixture is a regression snapshot of the oracle on the tiny fp32 workload
(batch 1, seq 256, d_model 256, 4/2 heads, d_h 64, router 256->64->3, EMA a=0.9,
L3 block 32, R=2, 16-bit codes; seed 0).  The definitions it follows are those of
"MKA: Memory-Keyed Attention for Efficient Long-Context Reasoning" (paper-notes
page, sections 1-4).  Re-run it only when a change to the oracle's arithmetic is
justified by a passage of the pages, and say which in the commit.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from fastmka_inputs import CONFIGS, make_inputs, to_f64  # noqa: E402

ROWS = [0, 1, 2, 31, 32, 33, 63, 64, 100, 127, 128, 200, 255]


def compute():
    cfg = CONFIGS["tiny_f32"]
    inp = make_inputs(cfg)
    w = oracle.weights_f64(*(to_f64(t) for t in (inp.w_q, inp.w_k, inp.w_v, inp.w_r1, inp.w_r2, inp.hash_proj)))
    out = oracle.fastmka_prefill(to_f64(inp.x), w, cfg)
    return {
        "workload": cfg.name,
        "citation": "MKA: Memory-Keyed Attention for Efficient Long-Context Reasoning, paper-notes page §1-§4",
        "writer": "tests/golden/make_golden.py (oracle/ only)",
        "rows": ROWS,
        "lam": out["lam"][0, ROWS].tolist(),
        "idx": out["idx"][0, ROWS].tolist(),
        "x_codes": [int(c) for c in out["x_codes"][0, ROWS]],
        "summary_codes": [int(c) for c in out["summary_codes"][0]],
        "O_row_sums": out["O"][0, ROWS].sum(-1).tolist(),
        "O_first8": out["O"][0, ROWS, :8].tolist(),
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_f32_oracle.json"), "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote tiny_f32_oracle.json")
