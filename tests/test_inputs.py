"""The seeded input generator (CPU only)."""
import numpy as np

from tree_speculative_decoding_05_b200 import inputs


def test_splitmix64_reference_vector():
    # splitmix64 from state 0: published first outputs of the generator.
    got = [int(x) for x in inputs.raw_u64(np.uint64(0), 0, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 65504.0])
    got = inputs.to_bf16_bits(x)
    assert list(got) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000, 0x4780]
    assert np.array_equal(inputs.bf16_bits_to_f64(got)[:4], [1.0, 1.0, 1.015625, -2.5])


def test_normals_have_unit_moments():
    z = inputs.normal(inputs.stream_base(3, 1), 200_000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


def test_random_trees_respect_limits():
    for q in (9, 33, 65, 128):
        p = inputs.random_parents(1, 0, q)
        assert p[0] == -1 and all(0 <= p[i] < i for i in range(1, q))
        depth = np.zeros(q, int)
        for i in range(1, q):
            depth[i] = depth[p[i]] + 1
        assert depth.max() <= inputs.MAX_DEPTH


def test_planted_chain_and_tokens():
    w = inputs.config(4, prefix_lens=[64])
    chain = w.forced_path[0]
    assert len(chain) == 16 and chain[0] == 0 and (np.diff(chain) > 0).all()
    for a, c in zip(chain[:-1], chain[1:]):
        assert w.parents[0, c] == a and w.target_tokens[0, a] == w.node_tokens[0, c]


def test_retrieve_pointers_enumerate_children_in_order():
    p = np.array([-1, 0, 0, 1, 0, 3], np.int32)
    first, sib = inputs.retrieve_pointers(p)
    assert list(first) == [1, 3, -1, 5, -1, -1]
    assert list(sib) == [-1, 2, 4, -1, -1, -1]


def test_workload_is_deterministic():
    a = inputs.config(0)
    b = inputs.config(0)
    assert np.array_equal(a.q_lat, b.q_lat) and np.array_equal(a.c_kv, b.c_kv)
    assert a.c_kv.shape == (1, 265, 512) and a.q_lat.shape == (1, 9, 64, 512)


def test_draft_batch_rows():
    """Drafts for the tree build: per (request, depth) row, K finite log-probs of a
    distribution whose remaining mass sits on the rest of the vocabulary, sorted best
    first, K distinct tokens; deterministic per seed; the documented top-1 mass."""
    d = inputs.draft_batch(7, 64, 15, 8)
    assert d.lp.shape == (64, 15, 8) and d.lp.dtype == np.float32
    assert d.tok.shape == (64, 15, 8) and d.tok.dtype == np.int32
    assert np.isfinite(d.lp).all() and (d.lp < 0).all()
    assert (np.diff(d.lp, axis=2) <= 0).all()
    head = np.log(np.exp(d.lp.astype(np.float64)).sum(axis=2))
    assert (head < 0).all()  # the tail keeps some mass
    assert ((d.tok >= 0) & (d.tok < inputs.VOCAB)).all()
    assert ((d.root_token >= 0) & (d.root_token < inputs.VOCAB)).all()
    for b in range(64):
        for r in range(15):
            assert len(set(d.tok[b, r].tolist())) == 8
    assert 0.5 < float(np.exp(d.lp[:, :, 0].astype(np.float64)).mean()) < 0.6
    again = inputs.draft_batch(7, 64, 15, 8)
    assert np.array_equal(again.lp, d.lp) and np.array_equal(again.tok, d.tok)
    other = inputs.draft_batch(8, 64, 15, 8)
    assert not np.array_equal(other.lp, d.lp)
    q = inputs.draft_batch(7, 4, 6, 4, quantum=0.5)
    assert np.array_equal(q.lp, np.round(q.lp * 2) / 2)
    u = inputs.draft_batch(7, 4, 6, 4, sort=False)
    assert (np.diff(u.lp, axis=2) > 0).any()


def test_draft_trees_have_the_documented_depth():
    """At budget 32 the drafts give trees of mean depth about 7, some reaching 15
    (built by the oracle's best-first expansion)."""
    import oracle
    d = inputs.draft_batch(7, 64, 15, 8)
    depth = oracle.tree_build(d.lp, d.tok, d.root_token, 33)["depth"].max(axis=1)
    assert 6.0 < float(depth.mean()) < 8.5 and int(depth.max()) == 15
