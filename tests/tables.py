"""The committed coefficient table the tests feed to the library as input.

tests/golden/polar_express_k4.json is written by
tests/golden/make_polar_express.py, which calls only oracle/ (the fp64 Remez
routine); the library never reads it, the tests pass its rows in."""
import json
import os

from muon_optimizer_step_02_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))
PE_TABLE = os.path.join(HERE, "golden", "polar_express_k4.json")


def polar_express_doc() -> dict:
    with open(PE_TABLE) as f:
        return json.load(f)


def polar_express_k4():
    return [tuple(r) for r in polar_express_doc()["coeffs"]]


def workload(idx: int) -> wl.Workload:
    """workloads.workload with the committed 4-step table for workload 3."""
    return wl.workload(idx, polar_express_k4() if idx == 3 else None)
