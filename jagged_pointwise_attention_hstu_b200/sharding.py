"""User sharding for data-parallel runs over several GPUs.

Users are independent units of the jagged forward: no attention crosses users
(blog "Generative Recommendation 16", item 1 "Ragged/Jagged kernel"), so a
global batch splits across ranks by whole users with no collective on the
data path.  The cost of a user is its forward flops -- the attention over its
visible pairs plus the two GEMMs over its tokens -- and the users go to ranks
longest-processing-time first (each user, in descending cost, to the rank
with the least cost so far), which keeps the slowest rank within 4/3 of the
best possible split.
"""
from __future__ import annotations

from typing import List

import numpy as np

from .workloads import Batch, offsets_from_lengths


def user_costs(lengths, num_candidates, d_model: int, num_heads: int, head_dim: int,
               mfalcon: bool) -> np.ndarray:
    """Forward flops of each user: 4 hd H (visible pairs) + 10 n d^2."""
    n = np.asarray(lengths, dtype=np.int64)
    c = np.asarray(num_candidates, dtype=np.int64) if mfalcon else np.zeros_like(n)
    n_h = n - c
    pairs = n_h * (n_h + 1) // 2 + c * (n_h + 1)
    return (4 * head_dim * num_heads * pairs + 10 * n * d_model * d_model).astype(np.float64)


def lpt_shards(costs, world: int) -> List[np.ndarray]:
    """Users per rank, longest processing time first.  Users are taken by
    descending cost (equal costs: lower index first) and each goes to the rank
    with the least total so far (equal totals: lower rank).  Each rank's users
    come back in ascending index order.  Deterministic."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = np.asarray(costs, dtype=np.float64)
    order = sorted(range(costs.shape[0]), key=lambda u: (-costs[u], u))
    load = [0.0] * world
    owned: List[List[int]] = [[] for _ in range(world)]
    for u in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owned[r].append(u)
        load[r] += float(costs[u])
    return [np.asarray(sorted(o), dtype=np.int64) for o in owned]


def shard_batch(batch: Batch, users) -> Batch:
    """The sub-batch of the given users (in the given order), weights shared."""
    users = np.asarray(users, dtype=np.int64)
    offs = np.asarray(batch.seq_offsets, dtype=np.int64)
    rows = (np.concatenate([np.arange(offs[u], offs[u + 1]) for u in users])
            if users.size else np.zeros(0, dtype=np.int64))
    lengths = np.asarray(batch.lengths, dtype=np.int64)[users]
    return Batch(lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
                 timestamps=np.asarray(batch.timestamps)[rows],
                 num_candidates=np.asarray(batch.num_candidates)[users],
                 x=np.asarray(batch.x)[rows], layers=batch.layers)


def concat_batches(batches: List[Batch]) -> Batch:
    """The users of several batches, packed one after another (the first
    batch's weights)."""
    lengths = np.concatenate([b.lengths for b in batches]).astype(np.int64)
    return Batch(lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
                 timestamps=np.concatenate([b.timestamps for b in batches]),
                 num_candidates=np.concatenate([b.num_candidates for b in batches]),
                 x=np.concatenate([b.x for b in batches], axis=0), layers=batches[0].layers)
