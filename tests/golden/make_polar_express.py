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

from oracle.polar_express import composed_band, polar_express_table  # noqa: E402

LO, HI, STEPS = 1e-3, 1.0, 4
# The design interval of each step tracks the true lower end of the singular
# values (no floor under it) and inflates the upper end by 5 %.  The margin
# keeps bf16 rounding from being amplified: on the 66-matrix 11L set (3 steps,
# seed 1337) the GPU's O differs from the fp64 oracle by at most 1.74e-2 with
# an inflation of 1.05, 2.23e-2 with 1.03 and 2.34e-2 with 1.01 (the
# tolerance is 2e-2); the plain greedy schedule (no margin) amplifies to about
# 6e-2 in a bf16 emulation.
CUSHION, INFLATE = 0.0, 1.05


def main():
    rows, intervals, design = polar_express_table(STEPS, LO, HI, CUSHION,
                                                  INFLATE)
    plain, _, _ = polar_express_table(STEPS, LO, HI)
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
        # the exact range of the composed schedule over [LO, HI]
        "band": list(composed_band(rows, LO, HI)),
        # the same for the plain greedy schedule (no margins): the best band
        # any 4 odd quintic steps reach on [LO, HI]
        "band_plain_greedy": list(composed_band(plain, LO, HI)),
    }
    with open(os.path.join(HERE, "polar_express_k4.json"), "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
