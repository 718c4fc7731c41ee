"""The tensor-core GEMM's work schedule, checked on the CPU: ``plan_check.cu`` includes the
kernel header's own Plan / unit_of / for_each_tile and is built by nvcc as a host program
(no GPU needed).  See that file for the properties checked."""
import os
import shutil
import subprocess

import pytest

from mask_only_logits_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))


def test_schedule_covers_every_tile_once(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "plan_check")
    cmd = [nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
           "--expt-relaxed-constexpr", "-I", build.CSRC, "-I", os.path.join(build.ROOT, "include"),
           "-o", exe, os.path.join(HERE, "plan_check.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    run = subprocess.run([exe, "3000"], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0 and run.stdout.startswith("ok"), run.stdout + run.stderr
