"""Host logic of the multi-GPU run, on CPU with two gloo ranks.

bench.py shards users across ranks (each rank draws its own seeded batch, no
collective on the data path), times every rank on its own device and reports
the whole job's units over the slowest rank's time.  Here two processes play
the ranks over gloo on 127.0.0.1."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch.distributed as dist

    import bench
    from jagged_pointwise_attention_hstu_b200 import workloads as wl

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    try:
        w = wl.WORKLOADS[0]
        batch = bench.rank_batch(w, rank, num_layers=1)
        digest = (batch.total_tokens, batch.num_users, float(np.abs(batch.x).sum()),
                  tuple(int(v) for v in batch.seq_offsets))
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        # a slower rank decides the job's time
        ms_local = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(ms_local, world)
        units = batch.total_tokens
        units_each = [None] * world
        dist.all_gather_object(units_each, units)
        units_all = bench.sum_over_ranks(units, world)
        value = bench.weak_scaling_value(units_all, ms_max)
        out.put((rank, digests, ms_max, value, units_each, units_all))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_users_and_take_the_max_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, dig0, ms0, v0, each0, all0), (r1, dig1, ms1, v1, each1, all1) = res
    assert (r0, r1) == (0, 1)
    # every rank saw the same set of batches, and the two ranks' users differ
    assert dig0 == dig1
    assert dig0[0] != dig0[1]
    # the slowest rank's time, on every rank
    assert ms0 == ms1 == 15.0
    # the job's units are every rank's units, counted once; same value on every rank
    assert each0 == each1
    assert all0 == all1 == sum(each0)
    assert v0 == v1 == pytest.approx(sum(each0) / 15e-3)


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.sum_over_ranks(7, 1) == 7
    assert bench.weak_scaling_value(1000, 2.0) == pytest.approx(5e5)


def _lpt_rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch.distributed as dist

    import bench
    from jagged_pointwise_attention_hstu_b200 import sharding
    from jagged_pointwise_attention_hstu_b200 import workloads as wl

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    try:
        w = wl.WORKLOADS[1]                     # Zipf lengths: skewed user costs
        batch = bench.rank_batch(w, rank, num_layers=1, world=world, shard="lpt")
        cost = float(sharding.user_costs(batch.lengths, batch.num_candidates, w.d_model,
                                         w.num_heads, w.head_dim, False).sum())
        mine = (batch.total_tokens, float(np.abs(batch.x).sum()), cost)
        every = [None] * world
        dist.all_gather_object(every, mine)
        out.put((rank, every))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_the_global_batch_by_lpt():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_lpt_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] == res[1][1]               # every rank saw the same split
    every = res[0][1]
    sys.path.insert(0, ROOT)
    import bench
    from jagged_pointwise_attention_hstu_b200 import sharding
    from jagged_pointwise_attention_hstu_b200 import workloads as wl
    w = wl.WORKLOADS[1]
    draws = [wl.make_batch(w, seed_offset=r, num_layers=1) for r in range(world)]
    glob = sharding.concat_batches(draws)
    # the two shards hold the global batch's tokens, each exactly once
    assert sum(e[0] for e in every) == glob.total_tokens
    assert sum(e[1] for e in every) == pytest.approx(float(np.abs(glob.x).sum()), rel=1e-9)
    # and the slowest rank carries less than with each rank on its own draw
    costs = [float(sharding.user_costs(d.lengths, d.num_candidates, w.d_model, w.num_heads,
                                       w.head_dim, False).sum()) for d in draws]
    assert max(e[2] for e in every) <= max(costs)
    total = sum(costs)
    assert max(e[2] for e in every) <= total / world * 1.05
