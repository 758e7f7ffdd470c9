"""Pins of the CPU oracle: checks against things fixed by the pages and by the
mathematics, each written independently of the oracle's own code.

Every function takes an `oracle.Oracle` and raises AssertionError on a mismatch,
so the same pins run against the real oracle (tests/test_oracle_*.py) and against
deliberately broken copies of it (tests/test_oracle_mutants.py).

Sources (page title, section):
  [Race Conditions] "Race Conditions, Buffer Aliasing, and the Architecture of a
      Native DDTree Inference Engine"
  [Foundation] "Building the Foundation: Architecting a Native CUDA DDTree
      Inference Engine"
  [Verdict] "The Microsecond Verdict: Validating a DDTree Kernel Fix Under Time
      Pressure"
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from tree_speculative_decoding_05_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
ATOL = 1e-12


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def rand_bf16(seed: int, tag: int, shape, scale: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    z = inputs.normal(inputs.stream_base(seed, 40 + tag, 0), n) * scale
    return inputs.to_bf16_bits(z).reshape(shape)


def f64(bits):
    return inputs.bf16_bits_to_f64(bits)


def ancestors_by_walk(parents, i):
    """Ancestor-or-self set of node i, by walking the parent chain."""
    out = {i}
    while parents[i] != -1:
        i = int(parents[i])
        out.add(i)
    return out


def dense_attention(qf, kf, vf, visible, scale):
    """Textbook masked softmax attention in float64 for one node's heads.
    qf [H, D], kf [T, D], vf [T, DV], visible bool [T]."""
    s = float(np.float32(scale)) * (qf @ kf.T)          # [H, T]
    s = np.where(visible[None, :], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return (e / z) @ vf, (m + np.log(z))[:, 0]


def small_problem(seed, B, Q, P, H, DL, DR, parents=None, zero_q=False):
    """Random bf16 problem with prefix lengths P (list) and given parents."""
    P = np.asarray(P, dtype=np.int32)
    cap = int(P.max()) + Q
    q_lat = rand_bf16(seed, 1, (B, Q, H, DL))
    q_rope = rand_bf16(seed, 2, (B, Q, H, DR))
    if zero_q:
        q_lat[:] = 0
        q_rope[:] = 0
    c_kv = rand_bf16(seed, 3, (B, cap, DL))
    k_rope = rand_bf16(seed, 4, (B, cap, DR))
    if parents is None:
        parents = np.stack([inputs.random_parents(seed, b, Q) for b in range(B)])
    return q_lat, q_rope, c_kv, k_rope, P, np.asarray(parents, dtype=np.int32)


# ---------------------------------------------------------------------------
# Mask
# ---------------------------------------------------------------------------

def pin_mask_golden(orc):
    """Hand-worked masks ([Foundation] "The Single-Threaded Heap Design")."""
    for case in _golden("mask_cases.json")["cases"]:
        parents = np.array([case["parents"]], dtype=np.int32)
        mask, depth, status = orc.build_mask(parents)
        want = np.array([[int(w) for w in row] for row in case["mask"]], dtype=np.uint64)
        assert status[0] == case["status"], case["name"]
        assert np.array_equal(mask[0], want), case["name"]
        assert np.array_equal(depth[0], np.array(case["depth"], dtype=np.int32)), case["name"]


def pin_mask_bruteforce(orc):
    """Every bit against an explicit parent-chain walk, incl. two-word rows."""
    for q in (1, 2, 9, 33, 63, 64, 65, 66, 128):
        for seed in range(3):
            parents = inputs.random_parents(500 + seed, q, q)
            mask, depth, status = orc.build_mask(parents[None, :])
            assert status[0] == 0
            for i in range(q):
                anc = ancestors_by_walk(parents, i)
                assert depth[0, i] == len(anc) - 1
                for a in range(q):
                    bit = (int(mask[0, i, a // 64]) >> (a % 64)) & 1
                    assert bit == (a in anc), (q, seed, i, a)
                for a in range(q, 64 * mask.shape[2]):
                    assert (int(mask[0, i, a // 64]) >> (a % 64)) & 1 == 0


def pin_mask_closed_forms(orc):
    """Chain -> lower triangular (with diagonal); star -> diagonal + column 0."""
    for q in (1, 5, 64, 65, 100):
        vis, depth, st = orc.visibility(inputs.chain_parents(q))
        assert st == 0
        assert np.array_equal(vis, np.tril(np.ones((q, q), dtype=np.uint8)))
        assert np.array_equal(depth, np.arange(q, dtype=np.int32))
        vis, depth, st = orc.visibility(inputs.star_parents(q))
        want = np.eye(q, dtype=np.uint8)
        want[:, 0] = 1
        assert st == 0 and np.array_equal(vis, want)
        assert np.array_equal(depth, (np.arange(q) > 0).astype(np.int32))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _all_rows(B, Q, H):
    return np.arange(B * Q * H, dtype=np.int64)


def pin_attn_chain_is_causal(orc):
    """A chain tree is ordinary causal attention over [prefix; tree block] with
    key = [c_kv | k_rope], query = [q_lat | q_rope], value = c_kv."""
    for (P, Q, H, DL, DR) in ((7, 6, 3, 32, 8), (40, 9, 64, 512, 64)):
        q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(
            11 + P, 1, Q, [P], H, DL, DR, parents=[inputs.chain_parents(Q)])
        scale = 1.0 / math.sqrt(192.0)
        out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, scale)
        T = P + Q
        kf = np.concatenate([f64(c_kv[0, :T]), f64(k_rope[0, :T])], axis=1)
        vf = f64(c_kv[0, :T])
        for i in range(Q):
            qf = np.concatenate([f64(q_lat[0, i]), f64(q_rope[0, i])], axis=1)
            visible = np.arange(T) <= P + i
            o_ref, lse_ref = dense_attention(qf, kf, vf, visible, scale)
            assert np.max(np.abs(out[0, i] - o_ref)) < ATOL
            assert np.max(np.abs(lse[0, i] - lse_ref)) < ATOL


def pin_attn_decode(orc):
    """q_len = 1 is single-token decode attention over all P + 1 rows."""
    for P in (0, 1, 5, 300):
        H, DL, DR = 4, 64, 16
        q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(
            90 + P, 2, 1, [P, P + 3], H, DL, DR, parents=[[-1], [-1]])
        scale = 0.125
        out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, scale)
        for b in range(2):
            T = int(Pv[b]) + 1
            kf = np.concatenate([f64(c_kv[b, :T]), f64(k_rope[b, :T])], axis=1)
            qf = np.concatenate([f64(q_lat[b, 0]), f64(q_rope[b, 0])], axis=1)
            o_ref, lse_ref = dense_attention(qf, kf, f64(c_kv[b, :T]), np.ones(T, bool), scale)
            assert np.max(np.abs(out[b, 0] - o_ref)) < ATOL
            assert np.max(np.abs(lse[b, 0] - lse_ref)) < ATOL


def pin_attn_tiny_bruteforce(orc):
    """Tiny problems (Q<=4, P<=3, H=2, d=8/4), every tree shape the generator makes,
    against a dense version whose visibility comes from parent-chain walks."""
    for seed in range(12):
        Q = 1 + seed % 4
        P = seed % 4
        B = 2
        q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(
            200 + seed, B, Q, [P, max(P - 1, 0)], 2, 8, 4)
        scale = 0.3
        out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, scale)
        for b in range(B):
            Pb = int(Pv[b])
            T = Pb + Q
            kf = np.concatenate([f64(c_kv[b, :T]), f64(k_rope[b, :T])], axis=1)
            for i in range(Q):
                anc = ancestors_by_walk(parents[b], i)
                visible = np.array([j < Pb or (j - Pb) in anc for j in range(T)])
                qf = np.concatenate([f64(q_lat[b, i]), f64(q_rope[b, i])], axis=1)
                o_ref, lse_ref = dense_attention(qf, kf, f64(c_kv[b, :T]), visible, scale)
                assert np.max(np.abs(out[b, i] - o_ref)) < ATOL
                assert np.max(np.abs(lse[b, i] - lse_ref)) < ATOL


def pin_attn_probs(orc):
    """Weights are exactly 0 on masked rows, non-negative, and sum to 1."""
    B, Q, H = 2, 17, 3
    q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(7, B, Q, [20, 5], H, 16, 8)
    out, lse, probs = orc.attn_rows(q_lat, q_rope, c_kv, k_rope, Pv, parents, 0.2,
                                    _all_rows(B, Q, H), want_probs=True)
    for r in range(B * Q * H):
        b, i = r // (Q * H), (r // H) % Q
        Pb = int(Pv[b])
        anc = ancestors_by_walk(parents[b], i)
        T = Pb + Q
        for j in range(probs.shape[1]):
            visible = j < T and (j < Pb or (j - Pb) in anc)
            if not visible:
                assert probs[r, j] == 0.0
            else:
                assert probs[r, j] > 0.0
        assert abs(probs[r].sum() - 1.0) < ATOL


def pin_attn_prefix_permutation(orc):
    """Outputs do not depend on the order of the prefix rows."""
    B, Q, H, P = 1, 5, 2, 13
    q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(31, B, Q, [P], H, 16, 8)
    out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, 0.25)
    perm = np.concatenate([np.random.RandomState(5).permutation(P), np.arange(P, P + Q)])
    out2, lse2 = orc.attn_all(q_lat, q_rope, c_kv[:, perm], k_rope[:, perm], Pv, parents, 0.25)
    assert np.max(np.abs(out - out2)) < ATOL and np.max(np.abs(lse - lse2)) < ATOL


def pin_attn_zero_query(orc):
    """q = 0: uniform weights, out = mean of the visible c_kv rows, lse = ln(count)."""
    B, Q, H, P = 1, 9, 2, 6
    q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(41, B, Q, [P], H, 16, 8, zero_q=True)
    out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, 0.7)
    v = f64(c_kv[0])
    for i in range(Q):
        anc = sorted(ancestors_by_walk(parents[0], i))
        rows = list(range(P)) + [P + a for a in anc]
        assert np.max(np.abs(out[0, i] - v[rows].mean(axis=0))) < ATOL
        assert np.max(np.abs(lse[0, i] - math.log(len(rows)))) < ATOL


def pin_attn_single_key(orc):
    """P = 0, q_len = 1: the root sees only itself, out = its c_kv row exactly and
    lse = its own scaled score."""
    H, DL, DR = 3, 32, 8
    q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(51, 1, 1, [0], H, DL, DR,
                                                             parents=[[-1]])
    scale = 0.4
    out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, scale)
    for h in range(H):
        assert np.array_equal(out[0, 0, h], f64(c_kv[0, 0]))
        s = float(np.float32(scale)) * (f64(q_lat[0, 0, h]) @ f64(c_kv[0, 0]) +
                                        f64(q_rope[0, 0, h]) @ f64(k_rope[0, 0]))
        assert abs(lse[0, 0, h] - s) < ATOL


def pin_attn_duplicate_keys(orc):
    """Every visible key twice: lse rises by ln 2, out is unchanged (root only)."""
    H, DL, DR, P = 2, 16, 8, 5
    q_lat, q_rope, c_kv, k_rope, Pv, parents = small_problem(61, 1, 1, [P], H, DL, DR,
                                                             parents=[[-1]])
    out, lse = orc.attn_all(q_lat, q_rope, c_kv, k_rope, Pv, parents, 0.3)
    idx = list(range(P)) + list(range(P)) + [P, P]   # prefix twice, root row twice
    ckv2 = c_kv[:, idx]
    kr2 = k_rope[:, idx]
    out2, lse2 = orc.attn_all(q_lat, q_rope, ckv2, kr2, np.array([2 * P + 1], np.int32),
                              parents, 0.3)
    assert np.max(np.abs(out2 - out)) < ATOL
    assert np.max(np.abs(lse2 - lse - math.log(2.0))) < ATOL


# ---------------------------------------------------------------------------
# Accept
# ---------------------------------------------------------------------------

def pin_accept_golden(orc):
    """Hand-worked walks ([Verdict] "The Crash That Demanded a Fix")."""
    for case in _golden("tree_accept_cases.json")["cases"]:
        arr = lambda k: np.array([case[k]], dtype=np.int32)
        path, alen, bonus, status = orc.tree_accept(arr("node_tokens"), arr("target_tokens"),
                                                    arr("next_token"), arr("next_sibling"))
        assert status[0] == case["status"], case["name"]
        assert alen[0] == case["accept_len"], case["name"]
        assert bonus[0] == case["bonus"], case["name"]
        assert np.array_equal(path[0], np.array(case["path"], np.int32)), case["name"]


def pin_accept_properties(orc):
    """On valid random trees the result is a root path whose every step matches the
    target, which cannot be extended, and whose bonus is the target after it."""
    w = inputs.make_workload("t", 77, 16, 33, [0] * 16, heads=1, d_latent=8, d_rope=8)
    path, alen, bonus, status = orc.tree_accept(w.node_tokens, w.target_tokens,
                                                w.next_token, w.next_sibling)
    assert (status == 0).all()
    for b in range(w.B):
        par = w.parents[b]
        p = path[b, :alen[b]]
        assert p[0] == 0 and (path[b, alen[b]:] == -1).all()
        for k in range(1, alen[b]):
            assert par[p[k]] == p[k - 1]
            assert w.node_tokens[b, p[k]] == w.target_tokens[b, p[k - 1]]
        cur = p[-1]
        kids = [c for c in range(w.q_len) if par[c] == cur]
        assert alen[b] == w.q_len or all(w.node_tokens[b, c] != w.target_tokens[b, cur] for c in kids)
        assert bonus[b] == w.target_tokens[b, cur]


# ---------------------------------------------------------------------------
# Compaction
# ---------------------------------------------------------------------------

def pin_compact_golden(orc):
    """Hand-worked gathers ([Race Conditions] "The Cache Compaction Problem")."""
    for case in _golden("kv_compact_cases.json")["cases"]:
        cap = case["capacity"]
        c_kv = np.array([[[10 * r, 10 * r + 1] for r in range(cap)]], dtype=np.uint16)
        k_rope = np.array([[[100 + r] for r in range(cap)]], dtype=np.uint16)
        ckv2, kr2, newp, status = orc.kv_compact(
            c_kv, k_rope, np.array([case["prefix"]], np.int32),
            np.array([case["path"]], np.int32), np.array([case["accept_len"]], np.int32),
            capacity=cap)
        assert status[0] == case["status"], case["name"]
        assert newp[0] == case["new_prefix"], case["name"]
        assert np.array_equal(ckv2[0], np.array(case["c_kv"], np.uint16)), case["name"]
        assert np.array_equal(kr2[0], np.array(case["k_rope"], np.uint16)), case["name"]


def pin_compact_closed_forms(orc):
    """Whole-block keep lists whose result has a closed form: row P + i takes the old
    row P + keep[i] for i < alen, every other row is unchanged ([Race Conditions] "The
    Cache Compaction Problem": the gather reads old rows, so every read precedes every
    write).  The reversed block makes every destination a source of another row; every
    second node reads ahead of each write."""
    Q, P, extra = 16, 5, 3
    cap = P + Q + extra
    rows = np.arange(cap, dtype=np.uint16)
    c_kv = np.stack([rows * 7 + 1, rows * 7 + 2], axis=-1)[None].astype(np.uint16)
    k_rope = (rows * 3 + 9)[None, :, None].astype(np.uint16)
    for keep in (list(range(Q - 1, -1, -1)), [2 * i for i in range(Q // 2)], [0], list(range(Q))):
        alen = len(keep)
        path = np.full((1, Q), -1, np.int32)
        path[0, :alen] = keep
        ckv2, kr2, newp, status = orc.kv_compact(c_kv, k_rope, np.array([P], np.int32), path,
                                                 np.array([alen], np.int32), capacity=cap)
        want_c, want_r = c_kv.copy(), k_rope.copy()
        for i, k in enumerate(keep):
            want_c[0, P + i] = c_kv[0, P + k]
            want_r[0, P + i] = k_rope[0, P + k]
        assert status[0] == 0 and newp[0] == P + alen, keep
        assert np.array_equal(ckv2, want_c) and np.array_equal(kr2, want_r), keep


# ---------------------------------------------------------------------------
# Tree build
# ---------------------------------------------------------------------------

def _num(v):
    return float(v)  # JSON holds "nan" / "-inf" as strings; float() reads both


def pin_build_golden(orc):
    """Hand-traced expansions ([Foundation] "The Single-Threaded Heap Design",
    "Tie-Breaking and Numerical Precision", "Assumptions Underlying the Design")."""
    for case in _golden("tree_build_cases.json")["cases"]:
        lp = np.array([[[_num(x) for x in row] for row in case["lp"]]], dtype=np.float32)
        r = orc.tree_build(lp, np.array([case["tok"]], np.int32),
                           np.array([case["root_token"]], np.int32), case["q_len"])
        for k in ("parents", "node_tokens", "depth", "next_token", "next_sibling"):
            assert r[k][0].tolist() == case[k], (case["name"], k)
        want = np.array([_num(x) for x in case["logw"]], dtype=np.float32)
        assert np.array_equal(r["logw"][0], want), case["name"]
        assert r["n_nodes"][0] == case["n_nodes"] and r["status"][0] == case["status"], case["name"]


def _int_lp(seed, D, K, lo=1, hi=4000):
    """Log-probs that are negative integers / 16 (exact in float32 and in every
    partial sum used here), sorted descending per depth."""
    s = inputs.stream_base(seed, 90, 0)
    mags = (lo + inputs.raw_u64(s, 0, D * K) % np.uint64(hi - lo)).astype(np.int64).reshape(D, K)
    mags.sort(axis=1)
    return -mags, (-mags).astype(np.float32) / 16.0


def pin_build_bruteforce(orc):
    """With every row of lp non-positive and sorted descending, a node never
    outweighs its parent or its previous sibling, so best-first expansion creates
    nodes in globally descending weight: the tree is the Q-1 heaviest nodes of
    the full K-ary tree of depth D.  Enumerate that full tree with exact integer
    weights and compare node set, creation order, parents, tokens, depth, logw."""
    import itertools
    checked = 0
    for seed in range(40):
        D, K, Q = 3 + seed % 2, 3, 12 + seed % 9
        ilp, lp = _int_lp(seed, D, K)
        tok = (1000 * np.arange(1, D + 1)[:, None] + np.arange(K)[None, :]).astype(np.int32)
        nodes = []  # (exact weight, rank path)
        for d in range(1, D + 1):
            for ranks in itertools.product(range(K), repeat=d):
                nodes.append((sum(int(ilp[k, r]) for k, r in enumerate(ranks)), ranks))
        nodes.sort(key=lambda x: -x[0])
        top = nodes[:Q - 1]
        weights = [w for w, _ in nodes[:Q]]
        if len(set(weights)) < len(weights):
            continue  # a tie at or inside the cut: the order is not fixed by weights alone
        checked += 1
        r = orc.tree_build(lp[None], tok[None], np.array([7], np.int32), Q)
        index = {(): 0}
        for n, (w, ranks) in enumerate(top, start=1):
            index[ranks] = n
            assert r["parents"][0, n] == index[ranks[:-1]]
            assert r["depth"][0, n] == len(ranks)
            assert r["node_tokens"][0, n] == tok[len(ranks) - 1, ranks[-1]]
            assert r["logw"][0, n] == np.float32(w / 16.0)
        assert r["n_nodes"][0] == Q and r["status"][0] == 0
    assert checked >= 20


def pin_build_closed_forms(orc):
    """topk = 1 gives a chain of min(D, Q-1) drafts; depth 1 gives a star of
    min(K, Q-1) children of the root in rank order."""
    for D, Q in ((5, 9), (9, 5), (1, 2)):
        lp = -np.arange(1, D + 1, dtype=np.float32)[:, None] / 4
        tok = np.arange(D, dtype=np.int32)[:, None] + 100
        r = orc.tree_build(lp[None], tok[None], np.array([3], np.int32), Q)
        n = 1 + min(D, Q - 1)
        assert r["n_nodes"][0] == n
        assert r["parents"][0, :n].tolist() == list(range(-1, n - 1))
        assert r["node_tokens"][0, 1:n].tolist() == list(range(100, 100 + n - 1))
        cum = np.cumsum(np.arange(1, n)) / 4  # exact quarters
        assert np.array_equal(r["logw"][0, 1:n], (-cum).astype(np.float32))
        assert (r["node_tokens"][0, n:] == -1).all() and (r["parents"][0, n:] == 0).all()
    for K, Q in ((6, 4), (3, 8)):
        lp = -np.arange(1, K + 1, dtype=np.float32)[None, :] / 8
        tok = np.arange(K, dtype=np.int32)[None, :] + 50
        r = orc.tree_build(lp[None], tok[None], np.array([3], np.int32), Q)
        n = 1 + min(K, Q - 1)
        assert r["n_nodes"][0] == n
        assert (r["parents"][0, 1:n] == 0).all()
        assert r["node_tokens"][0, 1:n].tolist() == list(range(50, 50 + n - 1))
        assert np.array_equal(r["logw"][0, 1:n], lp[0, :n - 1])
        assert r["next_token"][0, 0] == 1
        assert r["next_sibling"][0, 1:n].tolist() == list(range(2, n)) + [-1]


def pin_build_structure(orc):
    """On random float log-probs (any order): parents precede children, depth is the
    parent's plus one and at most D, each node's token is a token of its depth row,
    and next_token / next_sibling list each node's children in ascending index."""
    B, D, K, Q = 24, 6, 5, 33
    s = inputs.stream_base(5, 91, 0)
    lp = (inputs.normal(s, B * D * K) * 2.0).astype(np.float32).reshape(B, D, K)
    tok = np.arange(B * D * K, dtype=np.int32).reshape(B, D, K)
    r = orc.tree_build(lp, tok, np.arange(B, dtype=np.int32), Q)
    assert (r["status"] == 0).all() and (r["n_nodes"] == Q).all()
    for b in range(B):
        par, dep = r["parents"][b], r["depth"][b]
        assert par[0] == -1 and dep[0] == 0
        for i in range(1, Q):
            assert 0 <= par[i] < i and dep[i] == dep[par[i]] + 1 <= D
            assert r["node_tokens"][b, i] in tok[b, dep[i] - 1]
        for i in range(Q):
            kids = [c for c in range(1, Q) if par[c] == i]
            walk, c = [], r["next_token"][b, i]
            while c != -1:
                walk.append(int(c))
                c = r["next_sibling"][b, c]
            assert walk == kids


ALL_PINS = [
    pin_mask_golden, pin_mask_bruteforce, pin_mask_closed_forms,
    pin_attn_chain_is_causal, pin_attn_decode, pin_attn_tiny_bruteforce, pin_attn_probs,
    pin_attn_prefix_permutation, pin_attn_zero_query, pin_attn_single_key,
    pin_attn_duplicate_keys, pin_accept_golden, pin_accept_properties, pin_compact_golden,
    pin_compact_closed_forms,
    pin_build_golden, pin_build_bruteforce, pin_build_closed_forms, pin_build_structure,
]
