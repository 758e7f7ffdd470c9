"""The C ABI used from plain C programs (needs a B200): tests/c/ddt_abi_demo.c
is compiled with gcc against include/ddt.h and the in-tree libddt.so, then run;
it checks attention with zero queries against its closed form (the mean of the
visible rows, lse = ln of their count) and an accept walk on a chain;
tests/c/ddt_context_demo.c runs the library in two CUDA contexts of one device."""
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


def test_library_in_two_contexts(tmp_path):
    """tests/c/ddt_context_demo.c: the same split-KV call in two CUDA contexts of
    one device (created with the driver API), through ddt_verify_attn_noalloc and
    ddt_verify_attn with a workspace, then in the first context again.  What the
    library remembers per context (the no-allocation scratch address, the kernels'
    shared-memory limit) must be looked up afresh in a new context: all six
    results agree bit for bit, with every status OK and no fault flag."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ddt.library_path()
    cuda = _cuda_home()
    exe = tmp_path / "ddt_context_demo"
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"),
                           os.path.join(ROOT, "tests", "c", "ddt_context_demo.c"), "-o", str(exe),
                           "-L", os.path.dirname(lib), "-lddt", "-L",
                           os.path.join(cuda, "lib64"), "-L", os.path.join(cuda, "lib64", "stubs"),
                           "-lcudart", "-lcuda",
                           f"-Wl,-rpath,{os.path.dirname(lib)}:{os.path.join(cuda, 'lib64')}"])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 differing results, 0 non-finite outputs" in r.stdout
