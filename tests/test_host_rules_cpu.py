"""The scheduling rules that the router and the down kernels evaluate on the
same inputs (tensor-core K parts, candidate groups, row-stream stage
geometry) checked on the CPU over a grid of layer shapes: a host program
compiled with nvcc from the library's own headers, run without a GPU."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "intra_expert_activation_b200", "csrc")


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else shutil.which("nvcc")


@pytest.mark.timeout(300)
def test_shared_rules_stay_in_bounds(tmp_path):
    nvcc = _nvcc()
    if not nvcc:
        pytest.skip("nvcc not found")
    exe = str(tmp_path / "host_rules_check")
    cmd = [nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
           "--expt-relaxed-constexpr", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
           os.path.join(HERE, "host_rules_check.cu"), "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=240)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr
