"""Writes tests/golden/polar_express_k4.json: the 4-step Polar-Express-style
coefficient table used as the Newton-Schulz input of the 66-matrix K=4
workload.  Calls only oracle/ (the fp64 Remez routine).

PR #1396 "Record: Combined 3-Layer Recurrence + Parallel Residuals + Polar
Express + Brotli", table "Techniques Combined", row "Polar Express
Newton-Schulz": 4 minimax-optimal steps, coefficients not printed.

Run from the repository root:  python tests/golden/make_polar_express.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.polar_express import polar_express_table  # noqa: E402

LO, HI, STEPS = 1e-3, 1.0, 4
# Stability margins (see oracle/polar_express.py): without them the greedy
# minimax polynomials are steep enough that bf16 rounding of the working
# matrix is amplified past a 2e-2 relative error on small matrices.
CUSHION, INFLATE = 0.1, 1.02


def main():
    rows, intervals, design = polar_express_table(STEPS, LO, HI, CUSHION,
                                                  INFLATE)
    doc = {
        "source": "greedy minimax odd quintics (fp64 Remez), "
                  "oracle/polar_express.py",
        "citation": "PR #1396, table 'Techniques Combined', row 'Polar "
                    "Express Newton-Schulz' (4 minimax-optimal steps; "
                    "coefficients not printed on the page)",
        "initial_interval": [LO, HI],
        "cushion": CUSHION,
        "inflate": INFLATE,
        "steps": STEPS,
        "coeffs": [list(r) for r in rows],
        "intervals": [list(i) for i in intervals],
        "design_intervals": [list(i) for i in design],
    }
    with open(os.path.join(HERE, "polar_express_k4.json"), "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
