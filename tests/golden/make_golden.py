"""Writes oracle_regression.json: a frozen sample of the oracle's outputs.

Calls only ``oracle`` and ``pair_inputs``. The values are a regression anchor
for the oracle itself (any later change to its arithmetic shows up here and
must name the passage that justifies it); they are not a pin, since they come
from the oracle. Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import pair_inputs as pi  # noqa: E402

CASES = [
    # (N, seed, bf16, mask kind)
    (5, 101, False, "random"),
    (9, 102, True, "random"),
]
PICK = [(0, 0, 0), (1, 2, 5), (4, 3, 127), (2, 4, 64)]


def main():
    rows = []
    for N, seed, bf16, mask in CASES:
        d = pi.random_case(N, seed, bf16=bf16, mask=mask)
        for direction in ("outgoing", "incoming"):
            out = oracle.trimul(d, direction)
            rows.append({
                "N": N, "seed": seed, "bf16": bf16, "mask": mask, "direction": direction,
                "picks": [[i, j, c, float(out[i % N, j % N, c])] for i, j, c in PICK],
                "sum": float(out.sum()), "sum_abs": float(np.abs(out).sum()),
            })
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.json")
    with open(path, "w") as f:
        json.dump({"generator": "tests/golden/make_golden.py", "eps": 1e-5, "cases": rows}, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
