"""ddt_verify_attn_noalloc against ddt_verify_attn (needs a B200).

The allocation-free entry point serves callers that may not call cudaMalloc
(for example a plugin inside a framework that owns all device memory, or a
decode loop that cannot afford an allocation's synchronisation).  It must give
the same attention as the workspace-taking entry point while keeping its split
partials in the library's own static scratch array.  Two calls in a row, on
different inputs, check that what one call leaves in the shared array does not
leak into the next.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (DeviceWorkload, LSE_MAX_ABS, MAX_ABS, REL_L2, compare_attention,
                         out_format, rows_of, sample_rows)
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu

SPLITS = 4


def _noalloc_lib():
    lib = ddt.load()
    lib.ddt_verify_attn_noalloc.argtypes = [ctypes.POINTER(ddt.AttnArgs), ctypes.c_void_p]
    lib.ddt_verify_attn_noalloc.restype = ctypes.c_int32
    lib.ddt_verify_attn_noalloc_scratch_bytes.argtypes = []
    lib.ddt_verify_attn_noalloc_scratch_bytes.restype = ctypes.c_size_t
    return lib


def _close(got: torch.Tensor, want: torch.Tensor, tol_abs: float, tol_rel=None):
    g = got.double().cpu().numpy()
    r = want.double().cpu().numpy()
    assert np.isfinite(g).all()
    assert np.max(np.abs(g - r)) <= tol_abs
    if tol_rel is not None:
        assert np.linalg.norm(g - r) <= tol_rel * np.linalg.norm(r)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _noalloc_lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((4242, 4343)):
        w = inputs.make_workload("noalloc", seed, 2, 17, [3000 - 700 * call, 1800 + 500 * call])
        dw = DeviceWorkload(w)
        mask, _, _ = ddt.build_mask(dw.parents)
        max_prefix = int(w.prefix_lens.max())
        ref_out, ref_lse = ddt.verify_attn(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix,
                                           mask, w.softmax_scale, max_prefix=max_prefix,
                                           want_lse=True, num_splits=SPLITS)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        a = ddt._attn_args(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask,
                           w.softmax_scale, out, lse, max_prefix, SPLITS, None, None)
        assert lib.ddt_verify_attn_workspace_size(ctypes.byref(a)) > 0  # the split path is in use
        rc = lib.ddt_verify_attn_noalloc(ctypes.byref(a), stream)
        assert rc == ddt.DDT_OK, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        _close(out, ref_out, MAX_ABS, REL_L2)
        _close(lse, ref_lse, LSE_MAX_ABS)
        _check_oracle(out, lse, w, f"no-alloc call {call}")
    assert ddt.fault_flags(reset=True) == 0


def _check_oracle(out, lse, w, what):
    """Sampled rows (and the last node of every request) against the float64 oracle."""
    H = 64
    must = np.concatenate([np.arange((b + 1) * w.q_len * H - H, (b + 1) * w.q_len * H)
                           for b in range(w.B)])
    rows = sample_rows(w.B, w.q_len, H, 768, seed=w.seed, must=must)
    o_ref, l_ref = oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens,
                                    w.parents, w.softmax_scale, rows)
    compare_attention(rows_of(out, rows), o_ref, what, fmt=out_format(out))
    assert np.abs(lse.reshape(-1).cpu().numpy()[rows] - l_ref).max() <= LSE_MAX_ABS, what


def _auto_plan(lib, a):
    """The split count the automatic plan picks, and the one the no-alloc call is
    documented to use: the largest count below the plan whose partials fit the
    scratch array, else one split (which needs none)."""
    cap = int(lib.ddt_verify_attn_noalloc_scratch_bytes())
    planned = int(lib.ddt_verify_attn_num_splits(ctypes.byref(a)))
    if int(lib.ddt_verify_attn_workspace_size(ctypes.byref(a))) <= cap:
        return planned, planned
    for s in range(planned - 1, 1, -1):
        a.num_splits = s
        fits = int(lib.ddt_verify_attn_workspace_size(ctypes.byref(a))) <= cap
        a.num_splits = 0
        if fits:
            return planned, s
    return planned, 1


@pytest.mark.parametrize("B,Q,P,want", [(3, 33, 20000, 2), (4, 128, 32768, 1)])
def test_noalloc_automatic_plan_larger_than_its_scratch(B, Q, P, want):
    """num_splits = 0 on shapes whose planned partials exceed the 32 MiB array:
    3 x q_len 33 x prefix 20000 plans 4 splits (50 MB of partials) and must step
    down to 2 (25 MB); 4 x q_len 128 x prefix 32768 plans 2 splits (134 MB) and
    must fall back to one split.  The result equals ddt_verify_attn forced to
    that split count bit for bit, and the oracle within the tolerances."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _noalloc_lib()
    w = inputs.make_workload("noalloc-auto", 5150 + Q, B, Q, [P] * B, want_lse=True)
    dw = DeviceWorkload(w)
    mask, _, _ = ddt.build_mask(dw.parents)
    out = torch.full((B, Q, 64, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Q, 64), float("nan"), dtype=torch.float32, device="cuda")
    a = ddt._attn_args(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask,
                       w.softmax_scale, out, lse, P, 0, None, None)
    planned, used = _auto_plan(lib, a)
    assert used == want and planned > used
    assert int(lib.ddt_verify_attn_workspace_size(ctypes.byref(a))) > \
        int(lib.ddt_verify_attn_noalloc_scratch_bytes())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.ddt_verify_attn_noalloc(ctypes.byref(a), stream) == ddt.DDT_OK
    torch.cuda.synchronize()
    ref_out, ref_lse = ddt.verify_attn(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask,
                                       w.softmax_scale, max_prefix=P, want_lse=True,
                                       num_splits=used)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    _check_oracle(out, lse, w, f"no-alloc automatic B={B} Q={Q} P={P}")
    assert ddt.fault_flags(reset=True) == 0


def test_noalloc_rejects_forced_splits_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _noalloc_lib()
    cap = int(lib.ddt_verify_attn_noalloc_scratch_bytes())
    w = inputs.make_workload("noalloc-big", 7, 4, 33, [600] * 4)
    dw = DeviceWorkload(w)
    mask, _, _ = ddt.build_mask(dw.parents)
    out = torch.empty((w.B, w.q_len, 64, 512), dtype=torch.bfloat16, device="cuda")
    a = ddt._attn_args(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask,
                       w.softmax_scale, out, None, int(w.prefix_lens.max()), 64, None, None)
    need = w.B * w.q_len * 64 * 513 * 4 * 64
    assert need > cap
    rc = lib.ddt_verify_attn_noalloc(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ddt.DDT_ERR_UNSUPPORTED
