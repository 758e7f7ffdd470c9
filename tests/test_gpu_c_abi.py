"""The C ABI used from a plain C program (needs a B200): tests/c/ddt_abi_demo.c
is compiled with gcc against include/ddt.h and the in-tree libddt.so, then run;
it checks attention with zero queries against its closed form (the mean of the
visible rows, lse = ln of their count) and an accept walk on a chain."""
import os
import shutil
import subprocess

import pytest
import torch

from tree_speculative_decoding_05_b200 import ddt

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_home():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return os.path.dirname(os.path.dirname(os.path.realpath(nvcc)))


def test_c_program_drives_the_library(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ddt.library_path()
    cuda = _cuda_home()
    exe = tmp_path / "ddt_abi_demo"
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"),
                           os.path.join(ROOT, "tests", "c", "ddt_abi_demo.c"), "-o", str(exe),
                           "-L", os.path.dirname(lib), "-lddt", "-L",
                           os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                           f"-Wl,-rpath,{os.path.dirname(lib)}:{os.path.join(cuda, 'lib64')}"])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "accept_len 5 5" in r.stdout
