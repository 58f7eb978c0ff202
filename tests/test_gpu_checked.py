"""The device-checked build (MUON_DEVICE_CHECKS): the same kernels with every
decoded work item checked against its matrix's tile grid and every epilogue
store against its buffer before the access.  In a process of its own
(MUONB200_LIB selects the build), ragged shapes, both prologue variants, the
11L layer shapes and step counts 0..5 must match the oracle with no check
failing; and a work list whose last item lies outside its matrix (test hook
3, which only the checked build accepts) must be caught -- the step reports
MUON_ERR_DEVICE_CHECK, nothing is touched, and the next step is correct."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
from muon_optimizer_step_02_b200 import binding as B, workloads as wl
from gpu_harness import GpuMuon, check_step
assert B.lib().muon_device_checks() == 1
H = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
Q5 = [wl.FIXED_QUINTIC] * 5
shapes = [(1, 1), (7, 13), (13, 7), (300, 200), (200, 300), (129, 257), (2100, 100),
          (100, 2100), (511, 1025), (24, 9000)] + wl.gpt_layer_shapes(512, 8, 4, 64)
for k in (5, 1, 0):
    g = GpuMuon(wl.custom(shapes, H, [wl.FIXED_QUINTIC] * k, grad_std=1.0, wid=700 + k))
    for step in range(2):
        check_step(g, step, list(range(len(shapes))))
# an invalid work item is caught before any access
w = wl.custom([(256, 512), (512, 256), (300, 700)], H, Q5, grad_std=1.0, wid=710)
g = GpuMuon(w)
g.plan.set_fault(3)
g.step(g.grads(0))
assert g.plan.last_error() == B.MUON_ERR_DEVICE_CHECK
assert g.plan.last_error() == B.MUON_OK
g.plan.set_fault(0)
g2 = GpuMuon(w)
check_step(g2, 0, [0, 1, 2])
print("checked ok")
"""


def test_device_checked_build_passes_parity_and_catches_a_bad_item():
    from muon_optimizer_step_02_b200 import binding as B
    env = dict(os.environ, MUONB200_LIB=B.CHECKED_LIB_PATH)
    res = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + SCRIPT],
                         env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "checked ok" in res.stdout


def test_default_build_refuses_the_bad_item_hook():
    from muon_optimizer_step_02_b200 import binding as B
    from muon_optimizer_step_02_b200 import workloads as wl
    if B.lib().muon_device_checks():
        pytest.skip("this process runs the checked build")
    plan = B.MuonPlan([(64, 64)], 5)
    with pytest.raises(B.MuonError) as e:
        plan.set_fault(3)
    assert e.value.status == B.MUON_ERR_UNSUPPORTED
    plan.close()
