"""User sharding for data-parallel runs: LPT against the brute-force optimum,
costs against the oracle's count of visible pairs, and sub-batches against
the rows they come from."""
import itertools

import numpy as np
import pytest

import oracle
from jagged_pointwise_attention_hstu_b200 import sharding
from jagged_pointwise_attention_hstu_b200 import workloads as wl


def _makespan(costs, shards):
    return max(float(np.sum(np.asarray(costs)[s])) if len(s) else 0.0 for s in shards)


def test_lpt_within_grahams_bound_of_the_optimum():
    rng = np.random.default_rng(1)
    for trial in range(150):
        m = int(rng.integers(2, 4))
        n = int(rng.integers(1, 9))
        costs = rng.integers(1, 50, size=n).astype(np.float64)
        shards = sharding.lpt_shards(costs, m)
        # every user exactly once, each rank's users ascending
        got = np.sort(np.concatenate(shards))
        assert np.array_equal(got, np.arange(n))
        assert all(np.all(np.diff(s) > 0) for s in shards)
        best = min(max(sum(costs[u] for u in range(n) if a[u] == r) for r in range(m))
                   for a in itertools.product(range(m), repeat=n))
        assert _makespan(costs, shards) <= (4 / 3 - 1 / (3 * m)) * best + 1e-9


def test_lpt_is_deterministic_and_handles_more_ranks_than_users():
    costs = [5.0, 5.0, 1.0]
    assert [s.tolist() for s in sharding.lpt_shards(costs, 2)] == [[0, 2], [1]]
    assert [s.tolist() for s in sharding.lpt_shards(costs, 5)] == [[0], [1], [2], [], []]
    with pytest.raises(ValueError):
        sharding.lpt_shards(costs, 0)


@pytest.mark.parametrize("mfalcon", [False, True])
def test_costs_count_the_visible_pairs(mfalcon):
    lengths = np.array([1, 7, 300, 0, 129])
    ncand = np.array([0, 3, 100, 0, 129])
    c = sharding.user_costs(lengths, ncand, 64, 2, 32, mfalcon)
    mask = "mfalcon" if mfalcon else "causal"
    for b in range(lengths.shape[0]):
        pairs = oracle.visible_pairs([0, int(lengths[b])], [int(ncand[b])], mask)
        assert c[b] == 4 * 32 * 2 * pairs + 10 * int(lengths[b]) * 64 * 64


def test_shard_and_concat_keep_every_users_rows():
    w = wl.WORKLOADS[1]
    a = wl.make_batch(w, num_layers=1)
    b = wl.make_batch(w, num_layers=1, seed_offset=1)
    g = sharding.concat_batches([a, b])
    assert g.num_users == a.num_users + b.num_users
    assert np.array_equal(g.x[:a.total_tokens], a.x)
    users = np.array([40, 3, 0])
    s = sharding.shard_batch(g, users)
    for k, u in enumerate(users):
        lo, hi = int(g.seq_offsets[u]), int(g.seq_offsets[u + 1])
        r0, r1 = int(s.seq_offsets[k]), int(s.seq_offsets[k + 1])
        assert np.array_equal(s.x[r0:r1], g.x[lo:hi])
        assert np.array_equal(s.timestamps[r0:r1], g.timestamps[lo:hi])
        assert s.lengths[k] == g.lengths[u]
