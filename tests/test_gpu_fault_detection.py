"""Failure detection without a GPU fault (needs a B200).

Every wait in the library's kernels is bounded in time: a stalled barrier makes
the wait give up, set a bit in the library's fault word and return, so the
kernel ends and the context stays usable.  Here a self-test kernel waits (2 ms
at most) on a barrier that nothing completes; the host then reads the fault bit,
and a verify call afterwards must still be correct and clean."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import DeviceWorkload, compare_attention, out_format
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ddt.fault_flags(reset=True)
    gave_up = ddt.selftest_bounded_wait(2000)
    torch.cuda.synchronize()
    assert gave_up.item() == 1
    assert ddt.fault_flags(reset=True) == ddt.FAULT_WAIT_TIMEOUT
    assert ddt.fault_flags(reset=True) == 0  # the read above cleared it

    w = inputs.make_workload("after-fault", 3, 2, 9, [100, 37], want_lse=True)
    out, lse, status = DeviceWorkload(w).verify()
    torch.cuda.synchronize()
    assert (status.cpu().numpy() == 0).all()
    o_ref, _ = oracle.attn_all(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens, w.parents,
                               w.softmax_scale)
    compare_attention(out.float().cpu().numpy().reshape(-1, 512), o_ref.reshape(-1, 512),
                      "after the self-test", fmt=out_format(out))
    assert ddt.fault_flags(reset=True) == 0


def test_selftest_rejects_unbounded_limits():
    lib = ddt.load()
    assert lib.ddt_selftest_bounded_wait(0, None, None) == ddt.DDT_ERR_INVALID_ARG
    assert lib.ddt_selftest_bounded_wait(2_000_000, None, None) == ddt.DDT_ERR_INVALID_ARG
