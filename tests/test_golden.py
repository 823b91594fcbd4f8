"""The oracle and the seeded generator reproduce the frozen tiny fixture."""
import json
import os

import numpy as np

from tests.golden.make_tiny_fixture import compute

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_fixture_reproduces(oracle_lib):
    with open(os.path.join(HERE, "golden", "tiny_f32_oracle.json")) as f:
        fx = json.load(f)
    w, x, res = compute()
    assert fx["workload"] == w.name
    for k, v in fx["input_sums"].items():
        # tolerant of last-bit differences between BLAS builds in the QR of Pk/Pv
        assert abs(float(np.asarray(x[k].double().sum())) - v) <= 1e-9 * max(1.0, abs(v)), k
    np.testing.assert_array_equal(np.sort(res["idx"], axis=-1), np.array(fx["idx_sorted"]))
    np.testing.assert_allclose(res["out"], np.array(fx["out"]), rtol=0, atol=1e-9)
