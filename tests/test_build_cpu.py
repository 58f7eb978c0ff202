"""Register budget of the tensor-core kernel, checked on the CPU with ptxas
(no GPU needed).

The Newton-Schulz kernel launches with kNsRegsLaunch registers per thread
and then moves registers between its warpgroups with setmaxnreg: warpgroup 0
lowers its share to kNsRegsControl and the epilogue warpgroups raise theirs
to kNsRegsEpilogue.  An increase draws on the registers the block was
launched with, so the split is only safe if ptxas gives the kernel exactly
kNsRegsLaunch registers per thread and the shares add up to no more than
that; otherwise the increase would wait forever.  Both builds (default and
device-checked) must also compile without spills."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "muon_optimizer_step_02_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")


def _constant(src: str, name: str) -> int:
    m = re.search(rf"constexpr int {name} = (\d+);", src)
    assert m, f"{name} not found"
    return int(m.group(1))


def _ptxas_report(checked: bool, tmp_path) -> str:
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc is not available")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-Xptxas", "-v",
           "-I", INCLUDE, "-I", CSRC, "-c", "-o", str(tmp_path / "muon_api.o"),
           os.path.join(CSRC, "muon_api.cu")]
    if checked:
        cmd.insert(1, "-DMUON_DEVICE_CHECKS")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    return res.stdout + res.stderr


@pytest.mark.parametrize("checked", [False, True])
def test_newton_schulz_register_split_matches_the_launch(checked, tmp_path):
    src = open(os.path.join(CSRC, "k_ns_common.cuh")).read()
    epi_warps = _constant(src, "kEpiWarps")
    warp0 = _constant(src, "kEpiWarp0")
    launch = _constant(src, "kNsRegsLaunch")
    control = _constant(src, "kNsRegsControl")
    epilogue = _constant(src, "kNsRegsEpilogue")
    threads = 32 * (warp0 + epi_warps)
    # the shares fit what the block is launched with, which fits the SM
    assert 128 * control + 32 * epi_warps * epilogue <= threads * launch <= 65536
    assert control % 8 == 0 and epilogue % 8 == 0 and 24 <= control <= epilogue <= 256

    log = _ptxas_report(checked, tmp_path)
    m = re.search(r"Function properties for (_Z\w*ns_mega_pair_kernel\w*)\s*\n"
                  r"\s*(\d+) bytes stack frame, (\d+) bytes spill stores, "
                  r"(\d+) bytes spill loads\s*\n.*?Used (\d+) registers", log)
    assert m, "no ptxas report for the Newton-Schulz kernel"
    spill_stores, spill_loads, used = int(m.group(3)), int(m.group(4)), int(m.group(5))
    assert used == launch, f"launched with {used} registers per thread, split assumes {launch}"
    assert spill_stores == 0 and spill_loads == 0, "the Newton-Schulz kernel spills"
