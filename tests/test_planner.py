"""The split-KV planner behind ddt_verify_attn_num_splits / _workspace_size (host
logic, CPU only; without a device the planner assumes the B200's 148 SMs).

Pinned: the plans it picks for the five workloads (one split everywhere except the
single long request, which the measured split sweep on that workload put at four),
and the properties every plan keeps: a forced split count is used as given, the
workspace holds one fp32 partial output row of 512 plus its lse per query row and
split, and no plan has more splits than KV tiles or than 32."""
import ctypes

import pytest

from tree_speculative_decoding_05_b200 import ddt


def _plan(B, Q, max_prefix, num_splits=0):
    a = ddt.AttnArgs()
    a.B, a.q_len, a.num_heads, a.d_latent, a.d_rope = B, Q, 64, 512, 64
    a.capacity = max_prefix + Q
    a.max_prefix = max_prefix
    a.num_splits = num_splits
    lib = ddt.load()
    return (int(lib.ddt_verify_attn_num_splits(ctypes.byref(a))),
            int(lib.ddt_verify_attn_workspace_size(ctypes.byref(a))))


@pytest.mark.parametrize("B,Q,P,want", [(1, 9, 256, 1), (8, 33, 1024, 1), (64, 33, 4096, 1),
                                        (64, 65, 8192, 1), (1, 33, 32768, 4)])
def test_plans_of_the_workloads(B, Q, P, want):
    splits, ws = _plan(B, Q, P)
    assert splits == want
    assert ws == (0 if want == 1 else want * B * Q * 64 * 513 * 4)


@pytest.mark.parametrize("forced", [1, 2, 7])
def test_forced_split_count(forced):
    splits, ws = _plan(2, 17, 3000, forced)
    assert splits == forced
    assert ws == (0 if forced == 1 else forced * 2 * 17 * 64 * 513 * 4)


@pytest.mark.parametrize("B,Q,P", [(1, 1, 0), (1, 2, 127), (1, 128, 100000), (3, 9, 65536),
                                   (148, 33, 4096), (1000, 9, 300)])
def test_plan_bounds(B, Q, P):
    splits, _ = _plan(B, Q, P)
    tiles = (P + Q + 127) // 128
    assert 1 <= splits <= min(32, max(tiles, 1))


def test_whole_waves_are_not_split():
    """74 requests x 17 node pairs = 1258 work items = exactly 17 waves of the 74 CTA
    pairs: nothing to even out, so splitting only adds partials to write and merge.
    With fewer items a split can pay for itself by filling a ragged last wave (16
    requests: 272 items = 3.7 waves; four splits make 14.7)."""
    assert _plan(74, 33, 32768)[0] == 1
    assert _plan(16, 33, 32768)[0] > 1


def test_empty_batch_and_bad_shape():
    assert _plan(0, 33, 4096) == (1, 0)
    a = ddt.AttnArgs()
    a.B, a.q_len, a.num_heads, a.d_latent, a.d_rope = 1, 33, 32, 512, 64  # 32 heads: unsupported
    lib = ddt.load()
    assert lib.ddt_verify_attn_num_splits(ctypes.byref(a)) == 1
    assert lib.ddt_verify_attn_workspace_size(ctypes.byref(a)) == 0
