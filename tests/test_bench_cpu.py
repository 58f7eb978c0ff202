"""Host-side arithmetic of bench.py: the tensor-core work the Newton-Schulz
kernel issues per launch, against closed forms of the tiling."""
import types

import bench
from muon_optimizer_step_02_b200 import workloads as wl

PAIR_BLOCK = 2 * 256 * 256 * 64      # FLOPs of one 256 x 256 x 64 pair k-block


def _w(shapes, k):
    return types.SimpleNamespace(shapes=shapes, coeffs=[(3.4445, -4.775, 2.0315)] * k)


def _dense(shapes, k):
    return k * sum(4 * min(r, c) ** 2 * max(r, c) + 2 * min(r, c) ** 3
                   for r, c in shapes)


def test_single_pair_tile_issues_the_dense_count():
    # m = 256: one pair tile per product, nothing saved by symmetry
    for shape in ((256, 256), (256, 1024), (4096, 256)):
        assert bench.ns_issued_flops(_w([shape], 3)) == _dense([shape], 3)


def test_symmetry_saves_the_lower_tiles():
    # m = 512 = two 256-row blocks: the gram and the polynomial compute 3 of 4
    # pair tiles, the apply all of them
    m, n = 512, 2048
    dense_gram, dense_poly = 2 * m * m * n, 2 * m ** 3
    want = (dense_gram * 3 // 4 + dense_poly * 3 // 4 + dense_gram) * 5
    assert bench.ns_issued_flops(_w([(n, m)], 5)) == want


def test_ragged_shapes_round_up_to_whole_blocks():
    # 100 x 72: one pair tile, K blocks of 64 (two for the gram's n = 100,
    # two for the poly and apply's m = 72)
    assert bench.ns_issued_flops(_w([(100, 72)], 1)) == (2 + 2 + 2) * PAIR_BLOCK


def test_bench_workload_pair_k_blocks():
    # 11L x 512d: per layer 80 + 20 + 20 + 80 + 248 + 248 = 696 pair k-blocks
    # per step, 11 layers, 5 steps
    w = wl.workload(6)
    assert bench.ns_issued_flops(w) == 696 * 11 * 5 * PAIR_BLOCK
    assert bench.ns_issued_flops(w) < _dense(w.shapes, 5)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one
    JSON line with the contract's keys (small workload, short budget)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MUONB200_ORACLE_BUDGET_S="1")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference",
                          "--workload", "1", "--steps", "2", "--warmup", "1"],
                         cwd=root, env=env, capture_output=True, text=True,
                         timeout=300, check=True).stdout.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup",
                "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
