"""Writes tests/golden/config0_rows.json: oracle outputs on selected rows of the seeded tiny
workload (B=1, one head, T=256, d=64, fp32, G=4, seed 0).

The pages print no worked numeric example for kappa or yhat (the reproduction note's section
本地结果与边界 reports only the dense/HD max error of its own runs), so this fixture is a
regression record of the fp64 oracle, not a value from the pages.  It calls only oracle/ and
the shared seeded input generator.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from positive_quadratic_b200 import inputs as I  # noqa: E402

ROWS = [0, 1, 2, 63, 64, 127, 200, 255]


def main():
    p = I.config0()
    y, den = oracle.dense(p.q, p.k, p.v, p.group_id, p.L, p.G, p.eps, return_den=True)
    out = {
        "source": "oracle.dense on positive_quadratic_b200.inputs.config0(); regression record",
        "rows": ROWS,
        "yhat_first8": [[float(x) for x in y[0, 0, i, :8]] for i in ROWS],
        "normaliser": [float(den[0, 0, i]) for i in ROWS],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "config0_rows.json"),
              "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
