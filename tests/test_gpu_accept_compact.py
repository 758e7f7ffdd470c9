"""ddt_accept_compact against the oracle's accept walk followed by its compaction,
bit-exact (needs a B200).  The fused call must give exactly what the two steps
give in sequence ("Race Conditions, Buffer Aliasing, and the Architecture of a
Native DDTree Inference Engine", "The Cache Compaction Problem"; "The
Microsecond Verdict: Validating a DDTree Kernel Fix Under Time Pressure", "The
Crash That Demanded a Fix")."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import DeviceWorkload, i32
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _check(w, dw, in_place=False, prefix=None):
    P = w.prefix_lens if prefix is None else prefix
    p_dev = i32(P)
    outs = ddt.accept_compact(dw.node_tokens, dw.target_tokens, dw.next_token, dw.next_sibling,
                              dw.c_kv, dw.k_rope, p_dev,
                              new_prefix_lens=p_dev if in_place else None)
    torch.cuda.synchronize()
    path, alen, bonus, ast, newp, cst = (t.cpu().numpy() for t in outs)
    r_path, r_alen, r_bonus, r_ast = oracle.tree_accept(w.node_tokens, w.target_tokens,
                                                       w.next_token, w.next_sibling)
    c_ref, k_ref, p_ref, s_ref = oracle.kv_compact(w.c_kv, w.k_rope, P, r_path, r_alen,
                                                   capacity=w.capacity)
    assert np.array_equal(path, r_path) and np.array_equal(alen, r_alen)
    assert np.array_equal(bonus, r_bonus) and np.array_equal(ast, r_ast)
    assert np.array_equal(_u16(dw.c_kv), c_ref) and np.array_equal(_u16(dw.k_rope), k_ref)
    assert np.array_equal(cst, s_ref)
    assert np.array_equal(p_dev.cpu().numpy() if in_place else newp, p_ref)
    return r_alen


@pytest.mark.parametrize("cfg", [0, 1, 2, 4])
def test_accept_compact_configs(cfg):
    w = inputs.config(cfg)
    alen = _check(w, DeviceWorkload(w))
    if cfg == 4:
        assert alen[0] == 16


@pytest.mark.parametrize("Q", [2, 17, 65, 128])
def test_accept_compact_in_place_prefix(Q):
    w = inputs.make_workload("ac", 300 + Q, 12, Q, [0, 5, 64, 333] * 3, heads=1, d_latent=512,
                             d_rope=64, match_prob=0.9)
    _check(w, DeviceWorkload(w), in_place=True)


def test_accept_compact_bad_prefix_and_bad_pointers():
    w = inputs.make_workload("ac-bad", 41, 4, 9, [10, 10, 10, 10], heads=1, match_prob=0.9)
    w.next_sibling[1, 3] = 3        # cyclic sibling list: walk limit or a normal stop
    w.next_token[2, 0] = 77         # pointer out of range: bad index
    dw = DeviceWorkload(w)
    P = w.prefix_lens.copy()
    P[3] = w.capacity               # prefix past the capacity: no compaction
    _check(w, dw, prefix=P)
