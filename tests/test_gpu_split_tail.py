"""ddt_verify_attn_split_tail (prefix pass + tree-block pass + LSE merge) against
the oracle, and against the fused ddt_verify_attn (needs a B200).

The split follows the production design the pages planned ("Building the
Foundation: Architecting a Native CUDA DDTree Inference Engine", "Assumptions
Underlying the Design", item 2: a dense kernel for the long prefix, a custom
one only for the small tree tail); the result is the same attention, so the
tolerances are those of the fused kernel."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (DeviceWorkload, LSE_MAX_ABS, MAX_ABS, compare_attention, out_format,
                         rows_of, sample_rows)
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu


def _split_tail(dw, num_splits=0, want_lse=True):
    w = dw.w
    mask, _, _ = ddt.build_mask(dw.parents)
    od = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    status = torch.empty(w.B, dtype=torch.int32, device="cuda")
    out, lse = ddt.verify_attn(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask,
                               w.softmax_scale, max_prefix=int(w.prefix_lens.max()),
                               out_dtype=od, want_lse=want_lse, num_splits=num_splits,
                               status=status, split_tail=True)
    torch.cuda.synchronize()
    assert (status.cpu().numpy() == 0).all()
    return out, lse


def _check(w, rows=None, num_splits=0, what=""):
    dw = DeviceWorkload(w)
    out, lse = _split_tail(dw, num_splits)
    H = w.q_lat.shape[2]
    if rows is None:
        rows = np.arange(w.B * w.q_len * H, dtype=np.int64)
    o_ref, l_ref = oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens,
                                    w.parents, w.softmax_scale, rows)
    compare_attention(rows_of(out, rows), o_ref, what, fmt=out_format(out))
    l_gpu = lse.reshape(-1).cpu().numpy()[rows].astype(np.float64)
    assert np.max(np.abs(l_gpu - l_ref)) <= LSE_MAX_ABS, what
    # and against the fused pass: both are within MAX_ABS of the exact values, so
    # they differ by at most twice that (a bf16 ulp at |o| ~ 7 is already 0.03)
    f_out, f_lse, _ = dw.verify()
    torch.cuda.synchronize()
    assert float((f_out.float() - out.float()).abs().max()) <= 2 * MAX_ABS, what


@pytest.mark.parametrize("Q,P", [(1, 0), (2, 0), (9, 0), (3, 5), (9, 127), (17, 128),
                                 (33, 129), (65, 64), (128, 200), (33, 1000)])
def test_split_tail_small(Q, P):
    w = inputs.make_workload("st", 60 + Q + P, 2, Q, [P, max(P - 3, 0)])
    _check(w, what=f"Q={Q} P={P}")


@pytest.mark.parametrize("splits", [1, 2, 5])
def test_split_tail_forced_prefix_splits(splits):
    w = inputs.make_workload("st-splits", 78, 2, 9, [700, 1001], out_dtype="f32")
    _check(w, num_splits=splits, what=f"prefix splits={splits}")


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_split_tail_configs(cfg):
    w = inputs.config(cfg)
    H = 64
    n = w.B * w.q_len * H
    rows = None if cfg == 0 else sample_rows(w.B, w.q_len, H, 512, seed=10 + cfg,
                                             must=np.arange(n - 64, n))
    _check(w, rows=rows, what=f"config {cfg}")


def test_split_tail_requires_workspace():
    w = inputs.make_workload("st-ws", 5, 1, 9, [300])
    dw = DeviceWorkload(w)
    mask, _, _ = ddt.build_mask(dw.parents)
    out = torch.empty((1, 9, 64, 512), dtype=torch.bfloat16, device="cuda")
    a = ddt._attn_args(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask, w.softmax_scale,
                       out, None, 300, 0, None, None)
    lib = ddt.load()
    assert lib.ddt_verify_attn_split_tail_workspace_size(a) > 0
    assert lib.ddt_verify_attn_split_tail(a, None) == ddt.DDT_ERR_INVALID_ARG


def test_split_tail_whole_output_of_the_eight_request_workload():
    """The prefix / tail split over every output row of the 8 x q_len 33 x prefix
    1024 workload (16 896 rows), rel-L2 over the whole tensor."""
    from gpu_helpers import compare_whole

    w = inputs.config(1)
    dw = DeviceWorkload(w)
    out, lse = _split_tail(dw)
    compare_whole(out, lse, w, oracle, what="split tail, config 1 (whole output)")
