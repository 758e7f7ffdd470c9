"""The verify kernel's documented build options still compile for sm_100a, and a
combination that does not fit the shared memory is rejected at compile time
(CPU only: nvcc cross-compiles; nothing runs)."""
import concurrent.futures
import os
import shutil
import subprocess
import tempfile

import pytest

from tree_speculative_decoding_05_b200 import build

SRC = os.path.join(build.CSRC, "verify_attn.cu")

# (defines, expected to compile)
CASES = [
    ("-DDDT_VERIFY_K_STAGE_CHUNKS=1 -DDDT_VERIFY_V_KEYS=32", True),   # the earlier layout
    ("-DDDT_VERIFY_TILE_KEYS=256", True),                            # wide tiles
    ("-DDDT_VERIFY_WARP_MAP=10", True),                              # no idle warp
    ("-DDDT_VERIFY_K_STAGES=3", False),                              # 2 rings x 3 x 16 KB: too big
]


def _compile(defines: str):
    with tempfile.TemporaryDirectory() as d:
        cmd = [build.nvcc(), *build.ARCH_FLAGS, "-O1", "-std=c++17", "--expt-relaxed-constexpr",
               *defines.split(), "-I", build.INCLUDE, "-I", build.CSRC, "-c", SRC, "-o",
               os.path.join(d, "v.o")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return r.returncode, r.stdout + r.stderr


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_verify_build_options():
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(CASES)) as ex:
        results = list(ex.map(lambda c: _compile(c[0]), CASES))
    for (defines, ok), (rc, log) in zip(CASES, results):
        if ok:
            assert rc == 0, f"{defines}:\n{log[-2000:]}"
        else:
            assert rc != 0 and "shared memory budget" in log, f"{defines} should not fit:\n{log[-2000:]}"
