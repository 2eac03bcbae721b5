"""Writes tests/golden/oracle_small.json: a frozen output of the fp64 oracle
on a tiny seeded case, so that a later change to the oracle's arithmetic is
caught.  It calls only the oracle.  The pages print no numeric worked example
of the scan, so no stored value here comes from them; the hand-derived
example is half_decay_by_hand.json.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(20260101)
    b, L, H, P, N, G = 1, 6, 2, 2, 3, 1
    inp = {
        "x": rng.standard_normal((b, L, H, P)),
        "dt": rng.standard_normal((b, L, H)),
        "A": -rng.uniform(1.0, 16.0, H),
        "B": rng.standard_normal((b, L, G, N)),
        "C": rng.standard_normal((b, L, G, N)),
        "D": rng.standard_normal(H),
        "dt_bias": np.log(np.expm1(rng.uniform(1e-3, 0.1, H))),
        "init_state": 0.1 * rng.standard_normal((b, H, P, N)),
    }
    y, fin = oracle.load().ssd_fwd(**inp)
    out = {"about": __doc__.strip().splitlines()[0],
           "inputs": {k: v.tolist() for k, v in inp.items()},
           "y": y.tolist(), "final_state": fin.tolist()}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
