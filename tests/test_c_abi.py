"""The C ABI from plain C: tests/c/abi_step.c is compiled with gcc against include/dllm.h,
linked to libdllm.so and the CUDA runtime, and run (GPU).  Building it needs no GPU."""
import os
import shutil
import subprocess

import pytest

from mask_only_logits_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA = "/usr/local/cuda"


def _compile(out: str) -> None:
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("gcc not available")
    build.build()
    cmd = [cc, "-O2", "-std=c11", "-Wall", "-I", os.path.join(build.ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(HERE, "c", "abi_step.c"), "-o", out,
           "-L", build.PKG_DIR, "-ldllm", "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + build.PKG_DIR + ":" + os.path.join(CUDA, "lib64")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr


def test_c_program_compiles_against_the_header(tmp_path):
    _compile(str(tmp_path / "abi_step"))


@pytest.mark.gpu
def test_c_program_runs_a_decode_step(tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exe = str(tmp_path / "abi_step")
    _compile(exe)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.startswith("ok"), res.stdout + res.stderr
