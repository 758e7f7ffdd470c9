"""Placement of independent requests on GPUs.

Requests of the tree-verify step share nothing, so several GPUs split a batch by
request with no exchange on the data path.  A request's verify cost grows with
its cache rows (prefix + tree block), so a ragged batch is split by the
longest-processing-time-first rule (Graham, "Bounds on multiprocessing timing
anomalies", SIAM J. Appl. Math. 17(2), 1969): take requests in decreasing cost
and give each to the currently least-loaded GPU.  Its makespan is at most
4/3 - 1/(3m) times the optimum for m GPUs."""
from __future__ import annotations

import numpy as np


def request_costs(prefix_lens, q_len: int) -> np.ndarray:
    """Cost of each request: its cache rows (prefix + tree block)."""
    return np.asarray(prefix_lens, dtype=np.int64) + int(q_len)


def lpt_partition(costs, n_parts: int) -> list[np.ndarray]:
    """Request indices per part.  Requests in decreasing cost (ties: lower index
    first) go to the least-loaded part (ties: lower part index); each part's
    indices are returned in ascending order."""
    costs = np.asarray(costs, dtype=np.int64)
    if n_parts < 1:
        raise ValueError("n_parts must be >= 1")
    order = sorted(range(len(costs)), key=lambda b: (-int(costs[b]), b))
    load = [0] * n_parts
    parts: list[list[int]] = [[] for _ in range(n_parts)]
    for b in order:
        k = min(range(n_parts), key=lambda j: (load[j], j))
        parts[k].append(b)
        load[k] += int(costs[b])
    return [np.array(sorted(p), dtype=np.int64) for p in parts]
