"""The host list scheduler of the persistent Newton-Schulz kernel
(csrc/schedule.h), compiled with g++ and checked on CPU: every tile of every
(matrix, step, phase) appears exactly once, every item comes after every
item of the phase it reads (the kernel's deadlock-freedom condition), and
the simulated makespan is no worse than the plain phase-by-phase order."""
import os
import shutil
import subprocess
from collections import Counter, defaultdict

import pytest

import tables
from muon_optimizer_step_02_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "muon_optimizer_step_02_b200", "csrc")
CUDA_INC = "/usr/local/cuda/include"


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None or not os.path.isdir(CUDA_INC):
        pytest.skip("g++ or CUDA headers missing")
    out = str(tmp_path_factory.mktemp("sched") / "schedule_check")
    subprocess.run([gxx, "-O2", "-std=c++17", "-I", CSRC, "-I", CUDA_INC,
                    os.path.join(ROOT, "tests", "cpp", "schedule_check.cpp"),
                    "-o", out], check=True)
    return out


def run(exe, shapes, steps, clusters, group_bytes=-1.0, lag=0):
    """The list for a policy (group_bytes < 0: the library's default)."""
    inp = f"{len(shapes)} {steps} {clusters} {group_bytes} {lag}\n" + "".join(
        f"{r} {c}\n" for r, c in shapes)
    res = subprocess.run([exe], input=inp, capture_output=True, text=True,
                         check=True)
    lines = res.stdout.strip().split("\n")
    items = [tuple(int(v) for v in ln.split()) for ln in lines[:-2]]
    _, accepted, missed = lines[-2].split()
    # the device-side item check accepts every item and catches every
    # corruption of one
    assert int(accepted) == len(items) and int(missed) == 0
    makespan = float(lines[-1].split()[1])
    return items, makespan


def expected_tiles(r, c):
    m, n = min(r, c), max(r, c)
    t2, tn = -(-m // 256), -(-n // 256)
    sym = [(i, j) for i in range(t2) for j in range(i, t2)]
    app = [(i, j) for i in range(t2) for j in range(tn)]
    return sym, app, -(-m // 64), -(-n // 64)


def check(items, shapes, steps):
    # the completion count each item waits for: two per tile of the phase it
    # reads (0 for the first gram, which reads the prologue's output)
    for mat, mode, k, _ti, _tj, _kt, target in items:
        sym, app, _, _ = expected_tiles(*shapes[mat])
        want_t = 0 if (mode == 0 and k == 0) else \
            2 * (len(app) if mode == 0 else len(sym))
        assert target == want_t, (mat, mode, k, target, want_t)
    items = [it[:6] for it in items]
    # completeness
    want = Counter()
    for mat, (r, c) in enumerate(shapes):
        sym, app, ktm, ktn = expected_tiles(r, c)
        for k in range(steps):
            for t in sym:
                want[(mat, 0, k) + t + (ktn,)] += 1
                want[(mat, 1, k) + t + (ktm,)] += 1
            for t in app:
                want[(mat, 2, k) + t + (ktm,)] += 1
    assert Counter(items) == want
    # order: the last item of the read phase precedes the first reader
    last = {}
    for pos, (mat, mode, k, *_rest) in enumerate(items):
        last[(mat, mode, k)] = pos
    first = {}
    for pos, (mat, mode, k, *_rest) in enumerate(items):
        first.setdefault((mat, mode, k), pos)
    for (mat, mode, k), pos in first.items():
        if mode == 0 and k == 0:
            continue
        dep = (mat, 2, k - 1) if mode == 0 else (mat, mode - 1, k)
        assert last[dep] < pos, ((mat, mode, k), dep)


def phase_major_makespan(shapes, steps, clusters):
    """Simulated makespan of the plain order (per step: all gram tiles,
    then all poly, then all apply; longest first within a phase) under the
    same cost model and in-order-per-cluster execution."""
    def cost(r, c, mode, k):
        m, n = min(r, c), max(r, c)
        kt = -(-n // 64) if mode == 0 else -(-m // 64)
        extra = 12000.0 if (mode == 2 and k == steps - 1) else 0.0
        return 512.0 * kt + 3000.0 + extra
    order = []
    for k in range(steps):
        for mode in range(3):
            ph = []
            for mat, (r, c) in enumerate(shapes):
                sym, app, _, _ = expected_tiles(r, c)
                for _t in (app if mode == 2 else sym):
                    ph.append((cost(r, c, mode, k), mat, mode, k))
            ph.sort(key=lambda x: -x[0])
            order += ph
    done = defaultdict(float)
    remaining = Counter((mat, mode, k) for _, mat, mode, k in order)
    finish_at = {}
    cl = [0.0] * clusters
    # in-order per cluster; a dependency's finish is known once all its
    # items were simulated (they precede in the list)
    for pos, (c, mat, mode, k) in enumerate(order):
        q = pos % clusters
        dep = None if (mode == 0 and k == 0) else \
            ((mat, 2, k - 1) if mode == 0 else (mat, mode - 1, k))
        start = max(cl[q], finish_at.get(dep, 0.0) if dep else 0.0)
        cl[q] = start + c
        key = (mat, mode, k)
        done[key] = max(done[key], cl[q])
        remaining[key] -= 1
        if remaining[key] == 0:
            finish_at[key] = done[key]
    return max(cl)


@pytest.mark.parametrize("widx,steps,clusters", [(2, 5, 74), (3, 4, 74),
                                                 (4, 5, 74), (1, 5, 74),
                                                 (5, 5, 74)])
def test_schedule_valid_and_no_worse(exe, widx, steps, clusters):
    shapes = tables.workload(widx).shapes
    items, makespan = run(exe, shapes, steps, clusters)
    check(items, shapes, steps)
    assert makespan <= phase_major_makespan(shapes, steps, clusters) * 1.001


@pytest.mark.parametrize("group_mb,lag", [(15, 1), (15, 3), (31, 6), (0.001, 1)])
def test_wave_orders_are_valid(exe, group_mb, lag):
    """The wave orders (groups of consecutive matrices started `lag` phase
    slots apart) keep every dependency before its readers too."""
    for widx in (2, 4):
        shapes = tables.workload(widx).shapes
        items, _ = run(exe, shapes, 5, 74, group_mb * 2 ** 20, lag)
        check(items, shapes, 5)
    shapes = [(1, 1), (7, 13), (300, 200), (129, 257), (1000, 8), (513, 1025)]
    for steps, clusters in ((1, 1), (3, 2), (5, 7)):
        items, _ = run(exe, shapes, steps, clusters, group_mb * 2 ** 20, lag)
        check(items, shapes, steps)


def test_default_order_is_phase_major(exe):
    shapes = tables.workload(2).shapes
    assert run(exe, shapes, 5, 74) == run(exe, shapes, 5, 74, 1e30, 0)


def test_schedule_ragged_and_few_clusters(exe):
    shapes = [(1, 1), (7, 13), (300, 200), (129, 257), (1000, 8), (513, 1025)]
    for steps, clusters in ((1, 1), (3, 2), (5, 7)):
        items, _ = run(exe, shapes, steps, clusters)
        check(items, shapes, steps)
