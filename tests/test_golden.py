"""The oracle still reproduces its committed regression fixture (CPU only)."""
import json
import os

import numpy as np

import oracle


def test_oracle_matches_regression_fixture():
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")
    doc = json.load(open(path))
    H, W, dk, dv = doc["H"], doc["W"], doc["dk"], doc["dv"]
    N = H * W
    q = np.array(doc["q"]).reshape(1, N, 1, dk)
    k = np.array(doc["k"]).reshape(1, N, 1, dk)
    v = np.array(doc["v"]).reshape(1, N, 1, dv)
    g = np.array(doc["g"]).reshape(1, N, 1, dk)
    s0 = np.array(doc["s0"]).reshape(1, 1, dk, dv)
    for case in doc["cases"]:
        o, sf = oracle.gla_forward(q, k, v, g, H, W, case["direction"],
                                   s0 if case["init_state"] else None)
        np.testing.assert_allclose(o.ravel(), case["out"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sf.ravel(), case["final_state"], rtol=1e-12, atol=1e-14)
