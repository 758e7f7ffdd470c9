"""Request placement across GPUs (CPU only): every request placed exactly once, the
LPT rule followed step by step on a hand-worked case, and its makespan within
Graham's 4/3 - 1/(3m) bound of the brute-force optimum on small batches."""
import itertools

import numpy as np

from tree_speculative_decoding_05_b200 import inputs
from tree_speculative_decoding_05_b200.sharding import lpt_partition, request_costs


def test_hand_worked_lpt():
    # costs 7,6,5,4,3 on 2 parts: 7->A, 6->B, 5->B(6<7), 4->A(7<11), 3->A or B (11 vs 11: A)
    parts = lpt_partition([3, 7, 5, 6, 4], 2)
    assert [p.tolist() for p in parts] == [[0, 1, 4], [2, 3]]


def test_every_request_once_and_bound():
    rng = np.random.RandomState(0)
    for _ in range(40):
        n, m = rng.randint(1, 9), rng.randint(1, 4)
        costs = rng.randint(1, 50, size=n)
        parts = lpt_partition(costs, m)
        assert sorted(np.concatenate(parts).tolist()) == list(range(n))
        make = max(int(costs[p].sum()) for p in parts)
        best = min(max(sum(int(costs[b]) for b in range(n) if a[b] == k) for k in range(m))
                   for a in itertools.product(range(m), repeat=n))
        assert make <= (4 / 3 - 1 / (3 * m)) * best + 1e-9


def test_ragged_workload_is_balanced():
    P = inputs.ragged_prefixes(1003, 64, 256, 8192)
    parts = lpt_partition(request_costs(P, 65), 8)
    loads = [int(request_costs(P, 65)[p].sum()) for p in parts]
    assert max(loads) - min(loads) <= int(request_costs(P, 65).max())
