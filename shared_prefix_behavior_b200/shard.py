"""Sharding the ranking forward across GPUs (host side, no device work).

ReST's serving path (§3.5 of the paper's reading, shared-prefix serving) is
independent across users: a user's history, all of its request cutoffs and
all of their candidates form one unit that no other user's work reads. So
N GPUs split the users (one process per GPU), each runs rank_request on its
own packed sub-batch, and no collective is needed on the data path.

Users are assigned by longest-processing-time-first (LPT) on a cost model of
the forward's FLOPs: the causal encoder attention grows as L^2, the
projections and FFN as L, and the decoder as the candidate rows times their
cutoffs. Every rank computes the same plan from the same host arrays.
"""
from __future__ import annotations

import heapq
from typing import List, Sequence

import numpy as np


def user_costs(cu_seqlens: Sequence[int], req_user: Sequence[int], req_cutoff: Sequence[int],
               cu_cands: Sequence[int], d: int, n_layers: int, d_ff: int, K: int = 3) -> np.ndarray:
    """Forward FLOPs of each user (its encoder plus all of its requests' decoding)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    L = (cu[1:] - cu[:-1]).astype(np.float64)
    enc = n_layers * (2.0 * d * L * (L + 1) + L * (12.0 * d * d + 6.0 * d * d_ff))
    cost = enc.copy()
    cc = np.asarray(cu_cands, dtype=np.int64)
    for r, (u, c) in enumerate(zip(req_user, req_cutoff)):
        rows = K * float(cc[r + 1] - cc[r])
        cost[int(u)] += rows * (4.0 * d * c + 6.0 * d * d)
    return cost


def partition_users(costs: Sequence[float], world: int) -> List[List[int]]:
    """LPT: users by decreasing cost, each to the currently least-loaded rank.

    Deterministic (ties broken by user index, then rank index); each rank's
    users are returned in increasing order.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda u: (-float(costs[u]), u))
    heap = [(0.0, r) for r in range(world)]
    out: List[List[int]] = [[] for _ in range(world)]
    for u in order:
        load, r = heapq.heappop(heap)
        out[r].append(u)
        heapq.heappush(heap, (load + float(costs[u]), r))
    return [sorted(x) for x in out]


def shard_arrays(cu_seqlens, req_user, req_cutoff, cu_cands, users: Sequence[int]):
    """Index arrays of one rank's sub-batch.

    Returns (rows, cu_seqlens, req_user, req_cutoff, cu_cands, cand_rows,
    requests): the packed token rows and candidate rows of the global arrays
    that belong to `users`, and the sub-batch's own packed index arrays
    (users renumbered 0..len(users)-1 in the given order).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    users = list(users)
    rows = np.concatenate([np.arange(cu[u], cu[u + 1]) for u in users]) if users else np.zeros(0, np.int64)
    new_cu = np.zeros(len(users) + 1, dtype=np.int32)
    new_cu[1:] = np.cumsum([cu[u + 1] - cu[u] for u in users])
    remap = {u: i for i, u in enumerate(users)}
    cc = np.asarray(cu_cands, dtype=np.int64)
    reqs = [r for r in range(len(req_user)) if int(req_user[r]) in remap]
    cand_rows = np.concatenate([np.arange(cc[r], cc[r + 1]) for r in reqs]) if reqs else np.zeros(0, np.int64)
    new_cc = np.zeros(len(reqs) + 1, dtype=np.int32)
    new_cc[1:] = np.cumsum([cc[r + 1] - cc[r] for r in reqs])
    return (rows, new_cu, np.array([remap[int(req_user[r])] for r in reqs], dtype=np.int32),
            np.array([int(req_cutoff[r]) for r in reqs], dtype=np.int32), new_cc, cand_rows,
            np.array(reqs, dtype=np.int64))
