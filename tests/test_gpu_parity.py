"""CUDA path against the CPU oracle, through the C ABI (needs a B200).

Integer work (mask, accept, compaction) must match bit for bit; attention must
match the float64 oracle within max-abs 2e-2 and relative-L2 5e-3 (lse within
5e-3)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import oracle_pins
from gpu_helpers import (DeviceWorkload, LSE_MAX_ABS, compare_attention, compare_whole, i32,
                         out_format, rows_of, sample_rows)
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(autouse=True)
def _no_device_faults():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ddt.fault_flags(reset=True)
    yield
    torch.cuda.synchronize()
    assert ddt.fault_flags(reset=True) == 0, "a kernel hit a bounded-wait timeout"


# ---------------------------------------------------------------------------
# Mask
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("q", [1, 2, 9, 33, 63, 64, 65, 100, 128])
def test_build_mask_bit_exact(q):
    B = 6
    parents = np.stack([inputs.random_parents(900 + q, b, q) for b in range(B)])
    parents[3] = inputs.chain_parents(q)
    parents[4] = inputs.star_parents(q)
    if q > 2:
        parents[5, q - 1] = q - 1          # malformed: a node its own parent
    mask, depth, status = ddt.build_mask(i32(parents))
    m_ref, d_ref, s_ref = oracle.build_mask(parents)
    assert np.array_equal(mask.cpu().numpy().view(np.uint64), m_ref)
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    assert np.array_equal(status.cpu().numpy(), s_ref)


# ---------------------------------------------------------------------------
# Accept
# ---------------------------------------------------------------------------

def test_tree_accept_golden_cases():
    with open(os.path.join(GOLDEN, "tree_accept_cases.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        arr = lambda k: i32(np.array([case[k]]))
        path, alen, bonus, status = ddt.tree_accept(arr("node_tokens"), arr("target_tokens"),
                                                    arr("next_token"), arr("next_sibling"))
        assert status.item() == case["status"], case["name"]
        assert alen.item() == case["accept_len"], case["name"]
        assert bonus.item() == case["bonus"], case["name"]
        assert path.cpu().numpy()[0].tolist() == case["path"], case["name"]


@pytest.mark.parametrize("q,B", [(9, 1), (33, 8), (33, 64), (65, 64), (128, 37)])
def test_tree_accept_bit_exact(q, B):
    w = inputs.make_workload("acc", 300 + q, B, q, [0] * B, heads=1, d_latent=8, d_rope=8)
    nt, tt, fc, ns = w.node_tokens.copy(), w.target_tokens.copy(), w.next_token.copy(), w.next_sibling.copy()
    rng = np.random.RandomState(q)
    # a few malformed requests: random pointers (cycles likely) and out-of-range ones
    for b in range(0, B, 7):
        fc[b] = rng.randint(-1, q, size=q)
        ns[b] = rng.randint(-1, q, size=q)
        tt[b] = nt[b][rng.randint(0, q, size=q)]
    if B > 3:
        ns[3, rng.randint(q)] = q + 5
    got = ddt.tree_accept(i32(nt), i32(tt), i32(fc), i32(ns))
    ref = oracle.tree_accept(nt, tt, fc, ns)
    for g, r, name in zip(got, ref, ("path", "accept_len", "bonus", "status")):
        assert np.array_equal(g.cpu().numpy(), r), name


# ---------------------------------------------------------------------------
# Compaction
# ---------------------------------------------------------------------------

def _compact_case(B, Q, P, seed, kind):
    cap = int(max(P)) + Q + 3
    rng = np.random.RandomState(seed)
    c_kv = rng.randint(0, 65535, size=(B, cap, 512)).astype(np.uint16)
    k_rope = rng.randint(0, 65535, size=(B, cap, 64)).astype(np.uint16)
    path = np.full((B, Q), -1, dtype=np.int32)
    alen = np.zeros(B, dtype=np.int32)
    for b in range(B):
        n = int(rng.randint(1, Q + 1))
        if kind == "increasing":
            p = np.sort(rng.choice(np.arange(1, Q), size=n - 1, replace=False)) if Q > 1 else []
            p = np.concatenate([[0], p]).astype(np.int32)
        elif kind == "any":      # arbitrary (not a tree path): still race-free
            p = rng.randint(0, Q, size=n).astype(np.int32)
        else:                    # identity
            p = np.arange(n, dtype=np.int32)
        path[b, :n] = p
        alen[b] = n
    return c_kv, k_rope, np.asarray(P, np.int32), path, alen, cap


def _run_compact(c_kv, k_rope, P, path, alen, cap):
    ckv_t = torch.from_numpy(c_kv.view(np.int16)).cuda().view(torch.bfloat16)
    kr_t = torch.from_numpy(k_rope.view(np.int16)).cuda().view(torch.bfloat16)
    newp, status = ddt.kv_compact(ckv_t, kr_t, i32(P), i32(path), i32(alen))
    return (ckv_t.view(torch.int16).cpu().numpy().view(np.uint16),
            kr_t.view(torch.int16).cpu().numpy().view(np.uint16), newp.cpu().numpy(),
            status.cpu().numpy())


@pytest.mark.parametrize("kind", ["increasing", "any", "identity"])
@pytest.mark.parametrize("Q", [1, 9, 33, 65, 128])
def test_kv_compact_bit_exact(kind, Q):
    B = 16
    P = [0, 1, 7, 100] * 4
    c_kv, k_rope, Pv, path, alen, cap = _compact_case(B, Q, P, 7 * Q, kind)
    ref = oracle.kv_compact(c_kv, k_rope, Pv, path, alen, capacity=cap)
    got = _run_compact(c_kv, k_rope, Pv, path, alen, cap)
    for g, r, name in zip(got, ref, ("c_kv", "k_rope", "new_prefix", "status")):
        assert np.array_equal(g, r), name


def test_kv_compact_at_scale():
    """The benchmark's at-scale patterns on 512 requests x q_len 128: the reversed
    block (every row moves, each one onto a row another request row reads) and every
    second node, mixed with identity rows, bit for bit against the oracle."""
    B, Q = 512, 128
    c_kv, k_rope, Pv, path, alen, cap = _compact_case(B, Q, [256] * B, 91, "identity")
    for b in range(B):
        if b % 3 == 0:
            path[b, :] = np.arange(Q - 1, -1, -1); alen[b] = Q
        elif b % 3 == 1:
            path[b, :64] = 2 * np.arange(64); alen[b] = 64
    ref = oracle.kv_compact(c_kv, k_rope, Pv, path, alen, capacity=cap)
    got = _run_compact(c_kv, k_rope, Pv, path, alen, cap)
    for g, r, name in zip(got, ref, ("c_kv", "k_rope", "new_prefix", "status")):
        assert np.array_equal(g, r), name
    assert (ref[3] == 0).all()


def test_kv_compact_in_place_prefix_update():
    """new_prefix_lens = prefix_lens (the decode loop's in-place update): the
    slices of a request must all read the old prefix before it is overwritten.
    Every request of a 300-request batch moves rows; results bit for bit."""
    B, Q = 300, 65
    P = [int(x) for x in np.random.RandomState(5).randint(0, 400, size=B)]
    c_kv, k_rope, Pv, path, alen, cap = _compact_case(B, Q, P, 17, "any")
    ref = oracle.kv_compact(c_kv, k_rope, Pv, path, alen, capacity=cap)
    ckv_t = torch.from_numpy(c_kv.view(np.int16)).cuda().view(torch.bfloat16)
    kr_t = torch.from_numpy(k_rope.view(np.int16)).cuda().view(torch.bfloat16)
    prefix = i32(Pv)
    newp, status = ddt.kv_compact(ckv_t, kr_t, prefix, i32(path), i32(alen), new_prefix_lens=prefix)
    assert newp.data_ptr() == prefix.data_ptr()
    assert np.array_equal(ckv_t.view(torch.int16).cpu().numpy().view(np.uint16), ref[0])
    assert np.array_equal(kr_t.view(torch.int16).cpu().numpy().view(np.uint16), ref[1])
    assert np.array_equal(prefix.cpu().numpy(), ref[2]) and np.array_equal(status.cpu().numpy(), ref[3])


def test_kv_compact_race_pattern_and_errors():
    """keep = [0, 2, 3] (the racing pattern) plus malformed requests: every error
    status, and bad entries past the accepted length, which are never read."""
    B, Q = 8, 8
    c_kv, k_rope, Pv, path, alen, cap = _compact_case(B, Q, [5] * B, 3, "identity")
    path[0, :3] = [0, 2, 3]; alen[0] = 3
    alen[1] = 0                                  # bad length
    path[2, :2] = [0, 99]; alen[2] = 2            # bad index
    Pv[3] = cap                                  # prefix past capacity
    alen[4] = Q + 1                              # bad length (too long)
    Pv[5] = -1                                   # negative prefix
    path[6, :3] = [0, 2, 1]; path[6, 3:] = [-7, 99, 1000, -1, 8]; alen[6] = 3  # junk after alen
    path[7, :2] = [0, -1]; alen[7] = 2            # negative index
    ref = oracle.kv_compact(c_kv, k_rope, Pv, path, alen, capacity=cap)
    got = _run_compact(c_kv, k_rope, Pv, path, alen, cap)
    for g, r, name in zip(got, ref, ("c_kv", "k_rope", "new_prefix", "status")):
        assert np.array_equal(g, r), name
    assert list(ref[3]) == [0, 5, 2, 4, 5, 4, 0, 2]


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _check_attention(dw: DeviceWorkload, rows=None, num_splits=0, out_dtype=None, what=""):
    w = dw.w
    out, lse, status = dw.verify(num_splits=num_splits, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert (status.cpu().numpy() == 0).all()
    H = w.q_lat.shape[2]
    if rows is None:
        rows = np.arange(w.B * w.q_len * H, dtype=np.int64)
    o_ref, l_ref = oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens,
                                    w.parents, w.softmax_scale, rows)
    compare_attention(rows_of(out, rows), o_ref, what, fmt=out_format(out))
    l_gpu = lse.reshape(-1).cpu().numpy()[rows].astype(np.float64)
    assert np.max(np.abs(l_gpu - l_ref)) <= LSE_MAX_ABS, what
    return out, lse


@pytest.mark.parametrize("Q,P", [(1, 0), (1, 1), (2, 0), (3, 5), (9, 256), (5, 123), (9, 127),
                                 (17, 128), (33, 129), (33, 300), (65, 64), (128, 200)])
def test_verify_attn_small(Q, P):
    B = 2
    w = inputs.make_workload("small", 50 + Q + P, B, Q, [P, max(P - 3, 0)])
    _check_attention(DeviceWorkload(w), what=f"Q={Q} P={P}")


@pytest.mark.parametrize("splits", [1, 2, 3, 5, 8])
def test_verify_attn_forced_splits(splits):
    w = inputs.make_workload("splits", 77, 2, 9, [700, 1001], out_dtype="f32")
    _check_attention(DeviceWorkload(w), num_splits=splits, what=f"splits={splits}")


@pytest.mark.parametrize("tree", ["chain", "star"])
def test_verify_attn_tree_shapes(tree):
    w = inputs.make_workload("shape", 88, 3, 33, [0, 64, 250], tree=tree)
    _check_attention(DeviceWorkload(w), what=tree)


def test_verify_attn_ignores_cache_padding():
    """Cache rows past P + Q hold NaN: results must be unaffected."""
    w = inputs.make_workload("pad", 99, 2, 9, [100, 37], capacity=400)
    dw = DeviceWorkload(w)
    ref_out, ref_lse, _ = dw.verify()
    for b in range(w.B):
        T = int(w.prefix_lens[b]) + w.q_len
        dw.c_kv[b, T:] = float("nan")
        dw.k_rope[b, T:] = float("inf")
    out, lse, _ = dw.verify()
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_verify_attn_rejects_bad_prefix():
    w = inputs.make_workload("badp", 5, 3, 9, [10, 20, 30])
    dw = DeviceWorkload(w)
    dw.prefix[1] = w.capacity  # tree block would overrun the cache
    out, lse, status = dw.verify()
    torch.cuda.synchronize()
    assert status.cpu().numpy().tolist() == [0, ddt.REQ_BAD_PREFIX, 0]


def test_verify_attn_row_scaled_cache():
    """Rows scaled by U(0.5, 2): a wide score range that exercises the rescale."""
    w = inputs.make_workload("scaled", 123, 2, 65, [900, 2000], row_scale_range=(0.5, 2.0),
                             want_lse=True)
    _check_attention(DeviceWorkload(w), rows=sample_rows(2, 65, 64, 1500, seed=1), what="scaled")


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_verify_attn_configs(cfg):
    """The five workloads at full size, in the launch configuration the benchmark
    times (automatic split plan, the workload's output dtype, lse requested):
    EVERY output row against the float64 oracle, so every work item of the
    persistent schedule (request x node pair x KV split) is checked; relative L2
    over the whole output tensor."""
    w = inputs.config(cfg)
    dw = DeviceWorkload(w)
    out, lse, status = dw.verify()
    torch.cuda.synchronize()
    assert (status.cpu().numpy() == 0).all()
    del dw
    compare_whole(out, lse, w, oracle, what=f"config {cfg} (whole output)")


def test_verify_attn_whole_output_two_mask_words():
    """q_len 128 (two mask words per node, 64 node pairs) with ragged prefixes and
    an fp32 lse: every output row against the oracle."""
    P = inputs.ragged_prefixes(4242, 4, 0, 3000)
    w = inputs.make_workload("q128", 4242, 4, 128, P, want_lse=True,
                             row_scale_range=(0.5, 2.0))
    dw = DeviceWorkload(w)
    out, lse, status = dw.verify()
    torch.cuda.synchronize()
    assert (status.cpu().numpy() == 0).all()
    compare_whole(out, lse, w, oracle, what="4 x q128 ragged (whole output)")


def test_step_configs_accept_and_compact():
    """Config 2 and 4 continue with tree_accept and kv_compact: bit-exact."""
    for cfg in (2, 4):
        w = inputs.config(cfg)
        dw = DeviceWorkload(w)
        path, alen, bonus, st = ddt.tree_accept(dw.node_tokens, dw.target_tokens, dw.next_token,
                                                dw.next_sibling)
        ref = oracle.tree_accept(w.node_tokens, w.target_tokens, w.next_token, w.next_sibling)
        for g, r in zip((path, alen, bonus, st), ref):
            assert np.array_equal(g.cpu().numpy(), r)
        if cfg == 4:
            assert alen.item() == 16 and np.array_equal(ref[0][0, :16], w.forced_path[0])
        newp, cst = ddt.kv_compact(dw.c_kv, dw.k_rope, dw.prefix, path, alen)
        c_ref, k_ref, p_ref, s_ref = oracle.kv_compact(w.c_kv, w.k_rope, w.prefix_lens, ref[0],
                                                       ref[1])
        assert np.array_equal(dw.c_kv.view(torch.int16).cpu().numpy().view(np.uint16), c_ref)
        assert np.array_equal(dw.k_rope.view(torch.int16).cpu().numpy().view(np.uint16), k_ref)
        assert np.array_equal(newp.cpu().numpy(), p_ref) and np.array_equal(cst.cpu().numpy(), s_ref)


@pytest.mark.parametrize("seed", range(8))
def test_verify_attn_random_shapes(seed):
    """Seeded random shapes across the supported range: batch, q_len up to 128
    (two mask words), prefixes from 0 to a few thousand rows, either output dtype,
    forced or automatic split counts, fused or prefix/tail-split computation."""
    rng = np.random.RandomState(900 + seed)
    B = int(rng.randint(1, 5))
    Q = int(rng.choice([1, 2, 5, 17, 33, 64, 65, 100, 128]))
    P = rng.randint(0, 3000, size=B).astype(np.int32)
    out_dtype = "f32" if rng.rand() < 0.5 else "bf16"
    w = inputs.make_workload("fuzz", 900 + seed, B, Q, P, out_dtype=out_dtype, want_lse=True,
                             row_scale_range=(0.5, 2.0) if rng.rand() < 0.5 else None)
    dw = DeviceWorkload(w)
    splits = int(rng.choice([0, 0, 1, 2, 3, 7]))
    H = 64
    rows = sample_rows(B, Q, H, 1024, seed=seed, must=np.arange(B * Q * H - 64, B * Q * H))
    what = f"B={B} Q={Q} P={P.tolist()} {out_dtype} splits={splits}"
    _check_attention(dw, rows=rows, num_splits=splits, what=what)
    mask, _, _ = ddt.build_mask(dw.parents)
    od = torch.float32 if out_dtype == "f32" else torch.bfloat16
    out, lse = ddt.verify_attn(dw.q_lat, dw.q_rope, dw.c_kv, dw.k_rope, dw.prefix, mask,
                               w.softmax_scale, max_prefix=int(P.max()), out_dtype=od,
                               want_lse=True, num_splits=splits, split_tail=True)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens,
                                    w.parents, w.softmax_scale, rows)
    compare_attention(rows_of(out, rows), o_ref, what + " split", fmt=out_format(out))
    assert np.abs(lse.reshape(-1).cpu().numpy()[rows] - l_ref).max() <= LSE_MAX_ABS, what


def test_verify_attn_more_requests_than_the_length_ranking_holds():
    """Past 512 requests the kernel keeps the natural request order instead of
    ranking by length: 600 short ragged requests, sampled rows of every tenth."""
    B, Q = 600, 3
    P = inputs.ragged_prefixes(77, B, 0, 300)
    w = inputs.make_workload("many", 77, B, Q, P, heads=64, out_dtype="bf16")
    H = 64
    rows = np.concatenate([np.arange(b * Q * H, (b + 1) * Q * H, 7) for b in range(0, B, 10)])
    _check_attention(DeviceWorkload(w), rows=rows.astype(np.int64), what="600 requests")
