"""The no-allocation attention entry point against the handle path.

hstu_attention_noalloc is for callers that may not allocate device memory
while they run (the scratch lives in a fixed device array of the library).
Given the U, V, Q, K that hstu_layer_forward produced, it must give that
call's attention output bit for bit, call after call, while the configuration
and the batch change between calls -- up to the capacity limit of the array
-- and a warm call must leave the device's free memory unchanged."""
import pytest
import torch

from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# (lengths, candidates, d, H, time_log_div, time_buckets, n_norm, pos_clamp)
CASES = [
    ([300, 1, 0, 517, 129, 64], None, 256, 2, 0.301, 128, 0, 128),
    ([400, 77, 250], [50, 0, 10], 256, 4, 0.2, 64, 700, 64),
    # the capacity limit: HSTU_NOALLOC_MAX_TOKENS tokens, the row facts fill their slot
    ([8192] * 8, None, 256, 2, 0.301, 128, 8192, 1024),
]


def _case(idx, seed):
    lengths, ncand, d, H, div, nb, n_norm, clamp = CASES[idx]
    batch = wl.make_custom_batch(lengths, d, H, seed=seed, num_candidates=ncand,
                                 pos_buckets=clamp + 1, time_buckets=nb, weight_scale=0.05,
                                 rab_scale=0.5)
    cfg = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16,
                           compute_dtype=hstu.HSTU_DTYPE_BF16, n_norm=n_norm,
                           pos_buckets=clamp + 1, pos_clamp=clamp, time_buckets=nb,
                           time_log_div=div, ln_eps=1e-5, max_tokens=batch.total_tokens,
                           max_users=batch.num_users)
    mode = hstu.HSTU_MASK_CAUSAL if ncand is None else hstu.HSTU_MASK_MFALCON
    return batch, cfg, mode


def _handle_path(batch, cfg, mode):
    """U,V,Q,K and O of one hstu_layer_forward call (the existing entry point)."""
    T = batch.total_tokens
    handle = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, "bf16", "bf16", "cuda:0")
    out = torch.empty_like(db.x)
    handle.forward(db, out, mode)
    uvqk = handle.intermediate(hstu.HSTU_TENSOR_UVQK, T)
    av = handle.intermediate(hstu.HSTU_TENSOR_AV, T)
    torch.cuda.synchronize()
    assert handle.device_error() == 0
    handle.close()
    return db, uvqk, av


def _noalloc(cfg, db, uvqk, mode, ts=None):
    T = db.total_tokens
    av = torch.full((T, cfg.d_model), float("nan"), dtype=torch.float32, device="cuda:0")
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda:0")
    lp = db.layers[0]
    hstu.hstu_attention_noalloc(cfg, uvqk, T, db.seq_offsets, db.num_users,
                                db.timestamps if ts is None else ts, mode, db.num_candidates,
                                lp.rab_pos, lp.rab_time, av, err,
                                torch.cuda.current_stream())
    torch.cuda.synchronize()
    return av, int(err.item())


def test_noalloc_matches_the_handle_path_on_consecutive_calls():
    runs = [_case(0, 11), _case(1, 12)]
    refs = [_handle_path(*r) for r in runs]
    # two calls in a row per case, the cases alternating (tables, sizes and
    # masks change between consecutive calls)
    for rep in range(2):
        for (batch, cfg, mode), (db, uvqk, av_ref) in zip(runs, refs):
            av, err = _noalloc(cfg, db, uvqk, mode)
            assert err == 0
            assert torch.equal(av, av_ref), f"call {rep}: max diff {(av - av_ref).abs().max()}"


def test_noalloc_rejects_oversize_batches_before_any_launch():
    batch, cfg, mode = _case(0, 11)
    offs = torch.tensor([0, hstu.HSTU_NOALLOC_MAX_TOKENS + 1], dtype=torch.int32, device="cuda:0")
    with pytest.raises(hstu.HstuError) as ex:
        hstu.hstu_attention_noalloc(cfg, None, hstu.HSTU_NOALLOC_MAX_TOKENS + 1, offs, 1, None,
                                    mode, None, None, None, None)
    assert ex.value.status == hstu.HSTU_ERR_WORKSPACE


def test_noalloc_error_word_starts_at_zero_on_every_call():
    batch, cfg, mode = _case(0, 11)
    db, uvqk, av_ref = _handle_path(batch, cfg, mode)
    bad_ts = db.timestamps.clone()
    bad_ts[5] = bad_ts[4] - 1000      # decreasing inside the first user
    _, err = _noalloc(cfg, db, uvqk, mode, ts=bad_ts)
    assert err & hstu.HSTU_DEVERR_TIMESTAMPS
    av, err = _noalloc(cfg, db, uvqk, mode)
    assert err == 0
    assert torch.equal(av, av_ref)


def test_noalloc_at_the_capacity_limit_and_allocation_free_when_warm():
    batch, cfg, mode = _case(2, 13)
    assert batch.total_tokens == hstu.HSTU_NOALLOC_MAX_TOKENS
    db, uvqk, av_ref = _handle_path(batch, cfg, mode)
    av, err = _noalloc(cfg, db, uvqk, mode)      # warm call
    assert err == 0
    assert torch.equal(av, av_ref)
    out = torch.full_like(av, float("nan"))
    dev_err = torch.full((1,), -1, dtype=torch.int32, device="cuda:0")
    lp = db.layers[0]
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    hstu.hstu_attention_noalloc(cfg, uvqk, batch.total_tokens, db.seq_offsets, db.num_users,
                                db.timestamps, mode, db.num_candidates, lp.rab_pos, lp.rab_time,
                                out, dev_err, torch.cuda.current_stream())
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert int(dev_err.item()) == 0
    assert torch.equal(out, av_ref)


def test_noalloc_of_an_empty_batch():
    batch, cfg, mode = _case(0, 11)
    offs = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda:0")
    hstu.hstu_attention_noalloc(cfg, None, 0, offs, 0, None, hstu.HSTU_MASK_CAUSAL, None, None,
                                None, None, err, torch.cuda.current_stream())
    offs3 = torch.zeros(4, dtype=torch.int32, device="cuda:0")
    hstu.hstu_attention_noalloc(cfg, None, 0, offs3, 3, None, hstu.HSTU_MASK_CAUSAL, None, None,
                                None, None, err, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
