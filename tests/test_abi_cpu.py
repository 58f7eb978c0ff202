"""The C-ABI library builds, loads without a GPU, and exports every function
include/*.h declares.  Only calls that return before touching the GPU
(validation, constants) are made here."""
import ctypes
import glob
import os
import re

import pytest

from muon_optimizer_step_02_b200 import _build, binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return binding.lib()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^[A-Za-z_][\w \t\*]*?\b([a-z_][a-z0-9_]*)\s*\(",
                             text, flags=re.M):
            name = m.group(1)
            if name not in ("if", "while", "for", "return", "sizeof"):
                names.add(name)
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("muon_plan_create", "muon_plan_workspace_bytes",
                 "muon_step_batched", "ema_update_batched",
                 "muon_get_last_error", "muon_status_string",
                 "muon_plan_destroy"):
        assert must in names


def test_library_exports_every_declared_function(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_library_has_no_driver_or_torch_dependency():
    # Loads on a machine without libcuda: the driver entry point is resolved
    # at run time and the runtime is linked statically.
    import subprocess
    out = subprocess.run(["ldd", binding.LIB_PATH], capture_output=True,
                         text=True).stdout
    assert "libcuda.so" not in out
    assert "libtorch" not in out and "libc10" not in out


def test_constants(L):
    assert L.muon_abi_version() == 101
    import torch
    if not torch.cuda.is_available():
        # no plan can be created without a device, so nothing was allocated
        assert L.muon_device_allocation_count() == 0
    assert binding.status_string(0) == "ok"
    assert "timed out" in binding.status_string(-5)
    assert binding.status_string(-99) == "unknown status"
    assert L.muon_step_launches(5) == 2
    assert L.muon_step_launches(0) == 3
    assert L.muon_plan_step_launches(None, 5) == 0
    assert L.ema_update_launches(278) == 1
    assert L.ema_update_launches(321) == 2
    assert L.ema_update_launches(0) == 0
    assert L.muon_plan_workspace_bytes(None) == 0


def test_validation_returns_before_any_device_work(L):
    out = ctypes.c_void_p()
    rows = (ctypes.c_int32 * 1)(4)
    cols = (ctypes.c_int32 * 1)(4)
    assert L.muon_plan_create(None, cols, 1, 5, ctypes.byref(out)) == \
        binding.MUON_ERR_INVALID_ARG
    assert L.muon_plan_create(rows, cols, 0, 5, ctypes.byref(out)) == \
        binding.MUON_ERR_INVALID_ARG
    assert L.muon_plan_create(rows, cols, 1, 99, ctypes.byref(out)) == \
        binding.MUON_ERR_UNSUPPORTED
    bad = (ctypes.c_int32 * 1)(0)
    assert L.muon_plan_create(bad, cols, 1, 5, ctypes.byref(out)) == \
        binding.MUON_ERR_INVALID_ARG
    assert L.muon_step_batched(None, None, None, None, 0, None, 0, None) == \
        binding.MUON_ERR_INVALID_ARG
    assert L.ema_update_batched(None, None, None, 0, 0.5, None) == \
        binding.MUON_OK
    assert L.ema_update_batched(None, None, None, -1, 0.5, None) == \
        binding.MUON_ERR_INVALID_ARG
    assert L.ema_update_batched(None, None, None, 3, 0.5, None) == \
        binding.MUON_ERR_INVALID_ARG
    assert L.muon_get_last_error(None, None) == binding.MUON_ERR_INVALID_ARG
    assert L.muon_plan_set_timing(None, 1) == binding.MUON_ERR_INVALID_ARG
    L.muon_plan_destroy(None)


def test_ema_validation_catches_misalignment(L):
    e = (ctypes.c_void_p * 1)(0x1002)
    p = (ctypes.c_void_p * 1)(0x2000)
    n = (ctypes.c_int64 * 1)(8)
    assert L.ema_update_batched(e, p, n, 1, 0.9, None) == \
        binding.MUON_ERR_ALIGNMENT
    n2 = (ctypes.c_int64 * 1)(-1)
    assert L.ema_update_batched(e, p, n2, 1, 0.9, None) == \
        binding.MUON_ERR_INVALID_ARG
    n3 = (ctypes.c_int64 * 1)(8)
    assert L.ema_update_batched(e, p, n3, 1, float("nan"), None) == \
        binding.MUON_ERR_INVALID_ARG


def test_closed_plan_refuses_bound_calls(L):
    """A step bound to a plan reads the plan's handle at call time: once the
    plan is closed the call raises instead of passing a freed handle on."""
    plan = binding.MuonPlan.__new__(binding.MuonPlan)
    plan._h = None
    with pytest.raises(binding.MuonError) as e:
        plan._live_handle()
    assert e.value.status == binding.MUON_ERR_INVALID_ARG
    plan.close()                         # closing twice is harmless


def test_device_checked_build_loads_and_exports_the_same_calls(L):
    """The MUON_DEVICE_CHECKS build of the same sources (built by
    _build.build beside the default one) exports every declared function and
    reports itself; the default build reports 0."""
    assert L.muon_device_checks() == 0
    C = ctypes.CDLL(binding.CHECKED_LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(C, n)]
    assert not missing, missing
    C.muon_device_checks.restype = ctypes.c_int32
    assert C.muon_device_checks() == 1
    C.muon_status_string.restype = ctypes.c_char_p
    assert b"bounds check" in C.muon_status_string(-7)
