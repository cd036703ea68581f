"""The oracle still reproduces its frozen regression sample (tests/golden/oracle_regression.json)."""
import json
import os

import numpy as np

import oracle
import pair_inputs as pi

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_regression.json")


def test_oracle_regression_sample():
    with open(GOLDEN) as f:
        data = json.load(f)
    for row in data["cases"]:
        d = pi.random_case(row["N"], row["seed"], bf16=row["bf16"], mask=row["mask"])
        out = oracle.trimul(d, row["direction"])
        N = row["N"]
        for i, j, c, v in row["picks"]:
            assert abs(out[i % N, j % N, c] - v) <= 1e-12 * max(1.0, abs(v))
        np.testing.assert_allclose(out.sum(), row["sum"], rtol=1e-12)
        np.testing.assert_allclose(np.abs(out).sum(), row["sum_abs"], rtol=1e-12)
