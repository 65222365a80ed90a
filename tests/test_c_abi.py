"""A plain C program drives the library through include/moe_epilogue.h only.

The program is compiled and linked against libmoe_epilogue.so here (not gpu),
and run on the GPU (gpu)."""
import os
import shutil
import subprocess

import pytest

from moe_expert_epilogue_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "abi_smoke.c")
CUDA = os.path.dirname(os.path.dirname(shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"))


def _compile(tmp_path):
    lib = build.build()
    exe = tmp_path / "abi_smoke"
    cmd = ["gcc", "-std=c99", "-O1", SRC, "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), "-L", os.path.dirname(lib), "-lmoe_epilogue",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.dirname(lib)}",
           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", str(exe)]
    subprocess.run(cmd, check=True)
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
def test_c_program_runs_on_the_gpu(tmp_path, cuda_device):
    exe = _compile(tmp_path)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi_smoke: ok" in r.stdout
