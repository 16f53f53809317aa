"""Writes tests/golden/tiny_f32_rows.json from the CPU oracle alone.

This is a regression record of the oracle on the tiny fp32 workload (batch 1,
1024 tokens, 4 query heads / 1 KV head, d 64, block 64, top-k 4). The pages
print no worked example for this computation, so this file is not a pin of the
oracle against the pages; the pins are in tests/test_oracle_pins.py. It guards
against unintended changes to the oracle's arithmetic.

Run from the repository root: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle      # noqa: E402
import workloads   # noqa: E402

ROWS = [0, 63, 64, 255, 256, 700, 1023]


def main():
    w = workloads.tiny_f32()
    L = w.ctx[0]
    K = workloads.keys(w, 0, 0, L)
    V = workloads.values(w, 0, 0, L)
    Q = workloads.queries_prefill(w, 0, 0, L)
    pos = np.array(ROWS)
    r = oracle.forward(Q[ROWS], K, V, pos, w.block, w.top_k, w.softmax_scale)
    rec = {
        "source": "oracle/msa_oracle.cpp via tests/golden/make_golden.py (regression record, not a pin)",
        "workload": "tiny_f32",
        "rows": ROWS,
        "idx": r["idx"][:, 0].tolist(),
        "gap": [None if not np.isfinite(x) else float(x) for x in r["gap"][:, 0]],
        "lse": r["lse"].tolist(),
        "out_row_1023": r["out"][-1].tolist(),
        "centroid_block_3": r["centroids"][3, 0].tolist(),
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_rows.json"), "w") as f:
        json.dump(rec, f, indent=1)


if __name__ == "__main__":
    main()
