"""The multi-GPU path on the CPU: requests are independent, so N GPUs run N
replicas and the only cross-rank step is the timing reduction (max of the step
times, sum of the work).  Checked here with world_size 2 over gloo."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    w, r, _ = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    try:
        step_ms = [2.0, 3.5][rank]
        verify_ms = [1.5, 1.0][rank]
        mx = bench.reduce_max([step_ms, verify_ms], w, "cpu")
        sm = bench.reduce_sum([10.0 * (rank + 1)], w, "cpu")
        q.put((r, mx, sm))
    finally:
        dist.destroy_process_group()


def test_timing_reduction_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm in results:
        assert mx == [3.5, 1.5]          # each quantity's max over ranks
        assert sm == [30.0]


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.reduce_max([1.0, 2.0], 1, "cpu") == [1.0, 2.0]
    assert bench.reduce_sum([4.0], 1, "cpu") == [4.0]


def test_work_accounting_matches_definition():
    """FLOPs per verify call: 64 heads x 2 x (576 + 512) per visible key, where
    node i sees P + depth(i) + 1 keys (chain tree: depth(i) = i)."""
    import numpy as np

    import bench
    from tree_speculative_decoding_05_b200 import inputs
    parents = np.stack([inputs.chain_parents(5), inputs.star_parents(5)])
    prefix = np.array([10, 0], np.int32)
    f = bench.verify_flops(prefix, parents)
    vis = (10 * 5 + sum(range(1, 6))) + (1 + 2 * 4)
    assert f == 64 * 2 * 1088 * vis
    rows = np.arange(2 * 5 * 64)
    assert bench.flops_rows(prefix, parents, rows) == pytest.approx(f)


def _shard_worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import bench
    from tree_speculative_decoding_05_b200 import inputs
    from tree_speculative_decoding_05_b200.sharding import lpt_partition, request_costs

    bench.init_dist(world, "gloo")
    try:
        P = inputs.ragged_prefixes(1003, 64, 256, 8192)  # the ragged workload's prefixes
        mine = lpt_partition(request_costs(P, 65), world)[rank]
        counts = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(counts, torch.tensor([len(mine)]))
        n_max = int(max(c.item() for c in counts))
        padded = torch.full((n_max,), -1, dtype=torch.int64)
        padded[:len(mine)] = torch.from_numpy(mine)
        got = [torch.empty(n_max, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(got, padded)
        load = float(request_costs(P, 65)[mine].sum())
        q.put((rank, sorted(int(x) for g in got for x in g.tolist() if x >= 0), load))
    finally:
        dist.destroy_process_group()


def test_requests_split_longest_first_over_two_ranks():
    """Each rank derives the same longest-first partition and takes its part: the
    parts cover every request exactly once and their loads are balanced."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, union, _ in results:
        assert union == list(range(64))
    loads = [r[2] for r in results]
    assert abs(loads[0] - loads[1]) <= 8192 + 65


def _lpt_subset_worker(rank: int, world: int, port: int, q):
    """One rank of `bench.py --shard lpt` on the ragged workload's shape: the
    partition and the subset the benchmark takes (cheap per-request arrays: one
    head, 8-wide latent), then the request indices and prefix lengths of every
    rank gathered over gloo."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import torch
    import torch.distributed as dist

    import bench
    from tree_speculative_decoding_05_b200 import inputs
    from tree_speculative_decoding_05_b200.sharding import lpt_partition, request_costs

    bench.init_dist(world, "gloo")
    try:
        P = inputs.ragged_prefixes(1003, 64, 256, 8192)
        w = inputs.make_workload("ragged", 1003, 64, 65, P, heads=1, d_latent=8, d_rope=8,
                                 capacity=int(P.max()) + 65)
        part = lpt_partition(request_costs(w.prefix_lens, w.q_len), world)[rank]
        sub = inputs.subset(w, part)
        # the subset holds exactly the partition's requests, each array sliced alike
        ok = (sub.B == len(part) and np.array_equal(sub.prefix_lens, w.prefix_lens[part])
              and np.array_equal(sub.parents, w.parents[part])
              and np.array_equal(sub.c_kv, w.c_kv[part])
              and np.array_equal(sub.target_tokens, w.target_tokens[part]))
        n = torch.tensor([len(part)], dtype=torch.int64)
        counts = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(counts, n)
        n_max = int(max(int(c.item()) for c in counts))
        buf = torch.full((2, n_max), -1, dtype=torch.int64)
        buf[0, :len(part)] = torch.from_numpy(part)
        buf[1, :len(part)] = torch.from_numpy(sub.prefix_lens.astype(np.int64))
        got = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(got, buf)
        parts = [g[0, :int(c.item())].tolist() for g, c in zip(got, counts)]
        prefixes = [g[1, :int(c.item())].tolist() for g, c in zip(got, counts)]
        q.put((rank, ok, parts, prefixes))
    finally:
        dist.destroy_process_group()


def test_lpt_subsets_over_two_ranks_match_the_single_process_partition():
    """`--shard lpt` on two gloo ranks: every rank's subset is its share of the
    single-process longest-first partition; the shares are disjoint, cover the
    batch, and carry the right prefix lengths."""
    import numpy as np

    from tree_speculative_decoding_05_b200 import inputs
    from tree_speculative_decoding_05_b200.sharding import lpt_partition, request_costs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_lpt_subset_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    P = inputs.ragged_prefixes(1003, 64, 256, 8192)
    expect = [p.tolist() for p in lpt_partition(request_costs(P, 65), 2)]
    for rank, ok, parts, prefixes in results:
        assert ok, f"rank {rank}: subset arrays differ from the partition's requests"
        assert parts == expect                      # same partition on every rank
        flat = [b for part in parts for b in part]
        assert len(flat) == len(set(flat)) == 64    # disjoint
        assert sorted(flat) == list(range(64))      # covers the batch
        for part, pre in zip(parts, prefixes):
            assert pre == [int(P[b]) for b in part]
