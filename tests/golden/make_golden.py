"""Writes tests/golden/oracle_tiny.json from the fp64 oracle (and nothing else).

The pages print no worked example of the token mixer, so this fixture is a
regression record of the oracle itself: a 3x5 grid, dk=4, dv=3, all four scan
directions, with and without an initial state.  Inputs are stored as exact
fp16-representable values so the fixture does not depend on a random generator.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(20261202)
    H, W, dk, dv = 3, 5, 4, 3
    N = H * W
    f16 = lambda x: x.astype(np.float16).astype(np.float64)  # noqa: E731
    q = f16(rng.standard_normal((1, N, 1, dk)) * 0.5)
    k = f16(rng.standard_normal((1, N, 1, dk)))
    v = f16(rng.standard_normal((1, N, 1, dv)))
    g = f16(np.log(1.0 / (1.0 + np.exp(-rng.standard_normal((1, N, 1, dk)) * 2.0))) / 4.0)
    s0 = f16(rng.standard_normal((1, 1, dk, dv)) * 0.1)
    cases = []
    for d in range(4):
        for use_s0 in (False, True):
            o, sf = oracle.gla_forward(q, k, v, g, H, W, d, s0 if use_s0 else None)
            cases.append(dict(direction=d, init_state=use_s0, out=o.ravel().tolist(),
                              final_state=sf.ravel().tolist()))
    doc = dict(
        about="fp64 oracle regression fixture; written by tests/golden/make_golden.py",
        H=H, W=W, dk=dk, dv=dv, q=q.ravel().tolist(), k=k.ravel().tolist(),
        v=v.ravel().tolist(), g=g.ravel().tolist(), s0=s0.ravel().tolist(), cases=cases)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as fh:
        json.dump(doc, fh, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
