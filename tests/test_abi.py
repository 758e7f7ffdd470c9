"""The C ABI on the CPU: the library builds, loads, exports every symbol the
header declares, the ctypes mirror of ddt_attn_args matches the C layout, and
host-checkable argument errors are rejected before any launch (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from tree_speculative_decoding_05_b200 import build as ddt_build
from tree_speculative_decoding_05_b200 import ddt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ddt.h")


@pytest.fixture(scope="module")
def lib():
    ddt_build.build()
    return ddt.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DDT_API\s+[\w\s\*]+?\b(ddt_\w+)\s*\(", text)))


def test_header_declares_the_path_calls():
    names = declared_functions()
    for n in ("ddt_build_mask", "ddt_verify_attn", "ddt_tree_accept", "ddt_kv_compact",
              "ddt_tree_build", "ddt_accept_compact", "ddt_kv_write_block", "ddt_decode_step"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", ddt.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in ddt.EXPORTED_SYMBOLS:
        assert hasattr(lib, n)


@pytest.mark.parametrize("cname,pystruct", [("ddt_attn_args", ddt.AttnArgs),
                                             ("ddt_decode_args", ddt.DecodeArgs)])
def test_args_struct_layout_matches_c(tmp_path, cname, pystruct):
    src = tmp_path / "layout.c"
    fields = [f for f, _ in pystruct._fields_]
    body = "\n".join(f'  printf("{f} %zu\\n", offsetof({cname}, {f}));' for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "ddt.h"\nint main(void){\n'
                   f'  printf("sizeof %zu\\n", sizeof({cname}));\n{body}\n  return 0;\n}}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                           str(exe)])
    got = dict(line.split() for line in subprocess.check_output([str(exe)], text=True).splitlines())
    assert int(got["sizeof"]) == ctypes.sizeof(pystruct)
    for f in fields:
        assert int(got[f]) == getattr(pystruct, f).offset, f


def test_host_argument_checks(lib):
    V = ctypes.c_void_p
    # q_len out of range / negative batch: rejected before any CUDA call
    assert lib.ddt_build_mask(None, 1, 0, None, None, None, None) == ddt.DDT_ERR_UNSUPPORTED
    assert lib.ddt_build_mask(None, -1, 9, None, None, None, None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_build_mask(None, 1, 9, None, None, None, None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_build_mask(None, 0, 9, None, None, None, None) == ddt.DDT_OK
    assert lib.ddt_tree_accept(None, None, None, None, 1, 129, None, None, None, None,
                               None) == ddt.DDT_ERR_UNSUPPORTED
    assert lib.ddt_kv_compact(None, None, 0, 512, 0, 64, 10, None, None, None, 2, 9, None, None,
                              None) == ddt.DDT_ERR_INVALID_ARG
    a = ddt.AttnArgs(B=1, q_len=9, num_heads=32, d_latent=512, d_rope=64, capacity=300)
    assert lib.ddt_verify_attn(ctypes.byref(a), None) == ddt.DDT_ERR_UNSUPPORTED
    a.num_heads = 64
    assert lib.ddt_verify_attn(ctypes.byref(a), None) == ddt.DDT_ERR_INVALID_ARG  # null pointers
    # misaligned cache pointer
    fake = 0x10000
    a.prefix_lens = a.q_lat = a.q_rope = a.k_rope = a.mask = a.out = fake
    a.c_kv = fake + 2
    a.ckv_batch_stride, a.ckv_row_stride, a.kr_batch_stride, a.kr_row_stride = 300 * 512, 512, 300 * 64, 64
    assert lib.ddt_verify_attn(ctypes.byref(a), None) == ddt.DDT_ERR_INVALID_ARG
    a.c_kv = fake
    a.ckv_row_stride = 500  # shorter than a row
    assert lib.ddt_verify_attn(ctypes.byref(a), None) == ddt.DDT_ERR_INVALID_ARG
    a.ckv_row_stride = 512
    # the softmax scale must be positive and finite (checked before any launch)
    for bad in (0.0, -0.125, float("inf"), float("nan"), 3.0e38):
        a.softmax_scale = bad
        assert lib.ddt_verify_attn(ctypes.byref(a), None) == ddt.DDT_ERR_INVALID_ARG, bad
        assert lib.ddt_verify_attn_noalloc(ctypes.byref(a), None) == ddt.DDT_ERR_INVALID_ARG, bad
    a.softmax_scale = 0.0721
    a.B = 0
    assert lib.ddt_verify_attn(ctypes.byref(a), None) == ddt.DDT_OK
    # tree build: sizes, then null pointers; B = 0 is a no-op
    tb = lambda B, D, K, Q, p=None: lib.ddt_tree_build(p, p, p, B, D, K, Q, p, p, None, None, p, p,
                                                        None, None, None, None)
    assert tb(1, 15, 8, 129) == ddt.DDT_ERR_UNSUPPORTED
    assert tb(1, 15, 8, 0) == ddt.DDT_ERR_UNSUPPORTED
    assert tb(1, 0, 8, 33) == ddt.DDT_ERR_INVALID_ARG
    assert tb(1, 15, 0, 33) == ddt.DDT_ERR_INVALID_ARG
    assert tb(-1, 15, 8, 33) == ddt.DDT_ERR_INVALID_ARG
    assert tb(2, 15, 8, 33) == ddt.DDT_ERR_INVALID_ARG
    assert tb(0, 15, 8, 33) == ddt.DDT_OK
    assert lib.ddt_accept_compact(None, None, None, None, 1, 129, None, None, 0, 512, 0, 64, 300,
                                  None, None, None, None, None, None, None,
                                  None) == ddt.DDT_ERR_UNSUPPORTED
    assert lib.ddt_accept_compact(None, None, None, None, 1, 9, None, None, 0, 512, 0, 64, 300,
                                  None, None, None, None, None, None, None,
                                  None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_kv_write_block(None, None, 0, 512, 0, 64, 300, None, None, None, 1, 9, None,
                                  None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_kv_write_block(None, None, 0, 512, 0, 64, 300, None, None, None, 0, 9, None,
                                  None) == ddt.DDT_OK
    d = ddt.DecodeArgs()
    d.attn = ddt.AttnArgs(B=1, q_len=9, num_heads=64, d_latent=512, d_rope=64, capacity=300)
    d.depth_levels, d.topk = 15, 8
    assert lib.ddt_decode_step(ctypes.byref(d), None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_decode_step(None, None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_status_str(ddt.DDT_ERR_CUDA) == b"CUDA error"
    assert b"sm_100a" in lib.ddt_version()


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "tree_speculative_decoding_05_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "ddt_oracle" not in text and "oracle_" not in text, f
