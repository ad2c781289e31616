"""The C ABI from a plain C program (tests/c/abi_example.c): it compiles
against include/moe.h alone, links libmoe.so, and on a GPU runs prepare,
dispatch and combine and checks what their definitions fix."""

import os
import subprocess

import pytest

from combine_permute_b200 import _lib
from combine_permute_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile():
    build()
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_example")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA_HOME, "include"),
           os.path.join(ROOT, "tests", "c", "abi_example.c"), "-o", exe,
           "-L", lib_dir, "-l:libmoe.so", f"-Wl,-rpath,{lib_dir}",
           "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart",
           f"-Wl,-rpath,{os.path.join(CUDA_HOME, 'lib64')}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_program_compiles_and_links():
    assert os.path.exists(_compile())


@pytest.mark.gpu
def test_c_program_runs():
    exe = _compile()
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "c abi: ok" in r.stdout
