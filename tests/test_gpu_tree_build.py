"""ddt_tree_build against the oracle, bit-exact (needs a B200).

Every output of the build is integer or an exactly-specified float32 sum, so the
comparison is bit-for-bit: parents, tokens, depths, retrieve pointers, node
counts, status, the visibility words, and the float32 weights (including the
-inf of padding slots).  Inputs cover the pages' limits (budget <= 64, depth
<= 15; "Building the Foundation: Architecting a Native CUDA DDTree Inference
Engine", "The Single-Threaded Heap Design") and go past them to the library's
own (q_len <= 128), plus the edge cases the pages name (topk = 1 running out of
candidates, "Assumptions Underlying the Design", item 5) and equal weights
(insertion order, "Tie-Breaking and Numerical Precision")."""
import numpy as np
import pytest
import torch

import oracle
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu

FIELDS = ("parents", "node_tokens", "depth", "next_token", "next_sibling", "n_nodes", "status")


def _gpu_build(lp, tok, root, q_len):
    dev = torch.device("cuda")
    r = ddt.tree_build(torch.from_numpy(np.ascontiguousarray(lp, np.float32)).to(dev),
                       torch.from_numpy(np.ascontiguousarray(tok, np.int32)).to(dev),
                       torch.from_numpy(np.ascontiguousarray(root, np.int32)).to(dev), q_len)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in r.items()}


def _check(lp, tok, root, q_len):
    got = _gpu_build(lp, tok, root, q_len)
    want = oracle.tree_build(lp, tok, root, q_len)
    for k in FIELDS:
        assert np.array_equal(got[k], want[k]), k
    # float32 weights bit for bit (padding is -inf on both sides)
    assert np.array_equal(got["logw"].view(np.uint32), want["logw"].view(np.uint32))
    mask, _, _ = oracle.build_mask(want["parents"])
    assert np.array_equal(got["mask"].view(np.uint64), mask)
    return got


def _draft(seed, B, D, K, **kw):
    d = inputs.draft_batch(seed, B, D, K, **kw)
    return d.lp, d.tok, d.root_token


@pytest.mark.parametrize("B,D,K,Q", [(64, 15, 8, 33), (64, 15, 8, 65), (8, 15, 8, 9),
                                     (3, 15, 16, 128), (5, 4, 3, 33)])
def test_tree_build_matches_oracle(B, D, K, Q):
    g = _check(*_draft(2000 + Q, B, D, K), Q)
    assert (g["status"] == 0).all()


def test_tree_build_ties_follow_insertion_order():
    """Log-probs rounded to multiples of 0.5: many equal weights, so the pick order
    is decided by insertion order on both sides."""
    lp, tok, root = _draft(77, 32, 15, 8, quantum=0.5)
    _check(lp, tok, root, 65)
    lp = np.full((4, 6, 4), -1.0, np.float32)  # every weight ties
    _check(lp, tok[:4, :6, :4], root[:4], 40)
    lp = np.zeros((4, 6, 4), np.float32)  # +0 and -0 weights are equal weights
    lp[:, :, 1::2] = -0.0
    lp[1:, 2, :] = np.float32(-0.5)
    _check(lp, tok[:4, :6, :4], root[:4], 40)


def test_tree_build_unsorted_rows():
    _check(*_draft(78, 16, 10, 6, sort=False), 33)


def test_tree_build_chain_star_and_running_out():
    lp, tok, root = _draft(79, 4, 15, 8)
    g = _check(lp[:, :, :1], tok[:, :, :1], root, 33)  # topk 1: chain of 15, then padding
    assert (g["n_nodes"] == 16).all()
    g = _check(lp[:, :1, :], tok[:, :1, :], root, 33)  # depth 1: star of 8
    assert (g["n_nodes"] == 9).all()
    g = _check(lp[:, :2, :2], tok[:, :2, :2], root, 9)  # 1 + 2 + 4 nodes
    assert (g["n_nodes"] == 7).all()


def test_tree_build_extreme_sizes():
    lp, tok, root = _draft(80, 2, 140, 130)  # more rows and ranks than any build reads
    _check(lp, tok, root, 128)
    _check(lp, tok, root, 1)
    _check(lp, tok, root, 2)
    lp1, tok1, root1 = _draft(81, 1, 1, 1)
    _check(lp1, tok1, root1, 128)  # a single candidate, then 126 padding slots


@pytest.mark.parametrize("Q", [16, 17, 32, 33, 48, 49, 64, 65, 80, 81, 96, 97, 112, 113, 127])
def test_tree_build_every_key_register_count(Q):
    """The kernel is instantiated per number of candidate-key registers (1 to 8 per
    lane, the fewest holding 2 Q - 1 slots) and per nodes per lane; these budgets
    sit on both sides of every switch.  With D and K above Q every pick but the
    last inserts two candidates, so the slot count reaches its bound."""
    lp, tok, root = _draft(3000 + Q, 4, 130, 130)
    g = _check(lp, tok, root, Q)
    assert (g["n_nodes"] == Q).all()


def test_tree_build_non_finite_logprobs():
    lp, tok, root = _draft(82, 6, 15, 8)
    lp[1, 14, 7] = np.nan
    lp[3, 0, 0] = np.inf
    lp[4, 5, 2] = -np.inf
    g = _check(lp, tok, root, 33)
    assert g["status"].tolist() == [0, 6, 0, 6, 6, 0]
    assert g["n_nodes"].tolist() == [33, 1, 33, 1, 1, 33]


def test_tree_build_feeds_tree_accept():
    """The retrieve pointers drive ddt_tree_accept to the oracle's walk."""
    lp, tok, root = _draft(83, 16, 15, 8)
    g = _gpu_build(lp, tok, root, 33)
    rng = np.random.default_rng(5)
    target = np.where(rng.random((16, 33)) < 0.8, np.roll(g["node_tokens"], -1, axis=1),
                      rng.integers(0, 32000, (16, 33))).astype(np.int32)
    # make the greedy token after each node its first child's token most of the time
    for b in range(16):
        for i in range(33):
            c = g["next_token"][b, i]
            if c >= 0 and rng.random() < 0.7:
                target[b, i] = g["node_tokens"][b, c]
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    path, alen, bonus, st = ddt.tree_accept(t(g["node_tokens"]), t(target), t(g["next_token"]),
                                            t(g["next_sibling"]))
    want = oracle.tree_accept(g["node_tokens"], target, g["next_token"], g["next_sibling"])
    assert np.array_equal(path.cpu().numpy(), want[0])
    assert np.array_equal(alen.cpu().numpy(), want[1])
    assert (alen.cpu().numpy() > 1).any()


def test_tree_build_weights_that_overflow():
    """Finite log-probs whose sums overflow to -inf: the weights of whole subtrees
    become -inf and tie; both sides order them by insertion all the same."""
    lp, tok, root = _draft(84, 4, 12, 4)
    lp[:, 1:3, :] = np.float32(-3.0e38)  # depth-3 weights: -6e38 rounds to -inf
    lp[1, 0, 1:] = np.float32(-3.0e38)
    g = _check(lp, tok, root, 65)
    assert (g["status"] == 0).all() and (g["n_nodes"] == 65).all()
    assert (np.isinf(g["logw"]).sum(axis=1) >= 44).all()


def test_tree_build_golden_cases():
    """The hand-traced trees of the oracle's golden file, bit for bit on the GPU too
    (all-tied weights, the child-before-sibling insert, running out, a NaN, and the
    float32 parent-relative sibling weight that decides a tie)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tree_build_cases.json")
    for case in json.load(open(path))["cases"]:
        lp = np.array([[[float(x) for x in row] for row in case["lp"]]], dtype=np.float32)
        tok = np.array([case["tok"]], dtype=np.int32)
        g = _check(lp, tok, np.array([case["root_token"]], np.int32), case["q_len"])
        assert g["parents"][0].tolist() == case["parents"], case["name"]
