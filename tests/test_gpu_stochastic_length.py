"""GPU: Stochastic Length on the device against the oracle, bit for bit.

The kernels and the oracle take the same draws (u per user, a 32-bit key per
action) and decide "kept whole" by the same fp64 expression, so the new
offsets, the kept indices, the gathered rows and the timestamps must agree
exactly (ltzyclt blog on HSTU, section 5.1; blog "Generative Recommendation
16", item 2 "Stochastic Length")."""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu
from jagged_pointwise_attention_hstu_b200 import workloads as wl

pytestmark = pytest.mark.gpu

N_C, ALPHA = 776, 1.6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(lengths, u, keys, *, d=256, n_c=N_C, alpha=ALPHA, with_values=True, with_ts=True,
         seed=0):
    dev = "cuda:0"
    lengths = np.asarray(lengths, np.int64)
    offs = wl.offsets_from_lengths(lengths).astype(np.int32)
    T, B = int(offs[-1]), lengths.shape[0]
    rng = np.random.default_rng(seed)
    vals = torch.from_numpy(rng.normal(size=(max(T, 1), d)).astype(np.float32)).to(
        dev, torch.bfloat16)
    ts_np = np.sort(rng.integers(0, 2 ** 40, size=max(T, 1))).astype(np.int64)
    ts = torch.from_numpy(ts_np).to(dev)
    keys_np = np.asarray(keys, np.uint32)
    keys_d = torch.from_numpy(keys_np.view(np.int32).copy() if T else np.zeros(1, np.int32)).to(dev)
    u_d = torch.from_numpy(np.asarray(u, np.float64) if B else np.zeros(1)).to(dev)
    offs_d = torch.from_numpy(offs).to(dev)
    out_offs = torch.full((B + 1,), -1, dtype=torch.int32, device=dev)
    out_idx = torch.full((max(T, 1),), -1, dtype=torch.int64, device=dev)
    out_vals = torch.zeros_like(vals)
    out_ts = torch.full((max(T, 1),), -1, dtype=torch.int64, device=dev)
    scratch = torch.empty(hstu.hstu_stochastic_length_scratch_bytes(T, B), dtype=torch.uint8,
                          device=dev)
    err = torch.full((1,), -1, dtype=torch.int32, device=dev)
    hstu.hstu_stochastic_length(offs_d, B, T, u_d, keys_d, n_c, alpha,
                                vals if with_values else None, 2 * d,
                                ts if with_ts else None, out_offs, out_idx,
                                out_vals if with_values else None, out_ts if with_ts else None,
                                scratch, err, torch.cuda.current_stream())
    torch.cuda.synchronize()
    return dict(offs=offs, T=T, vals=vals, ts=ts_np, out_offs=out_offs.cpu().numpy(),
                out_idx=out_idx.cpu().numpy(), out_vals=out_vals, out_ts=out_ts.cpu().numpy(),
                err=int(err.item()))


def _check(res, lengths, u, keys, *, n_c=N_C, alpha=ALPHA, with_values=True, with_ts=True):
    ref_offs, ref_idx = oracle.stochastic_length(res["offs"], u, keys, n_c, alpha)
    assert res["err"] == 0
    assert np.array_equal(res["out_offs"], ref_offs)
    n = ref_idx.shape[0]
    assert np.array_equal(res["out_idx"][:n], ref_idx)
    if with_ts:
        assert np.array_equal(res["out_ts"][:n], res["ts"][ref_idx])
    if with_values and n:
        sel = torch.from_numpy(ref_idx).to(res["vals"].device)
        assert torch.equal(res["out_vals"][:n], res["vals"][sel])


def _keys(rng, T):
    return rng.integers(0, 2 ** 32, size=T, dtype=np.uint64).astype(np.uint32)


def test_mixed_lengths_bit_exact():
    rng = np.random.default_rng(11)
    lengths = [0, 1, 776, 777, 1500, 4096, 8192, 3000, 2, 5000, 1552, 8000]
    u = rng.random(len(lengths))
    u[7] = 0.0                  # a long user kept whole
    keys = _keys(rng, int(np.sum(lengths)))
    res = _run(lengths, u, keys, seed=1)
    _check(res, lengths, u, keys)
    # most long users are sampled, so the batch shrinks
    assert res["out_offs"][-1] < res["T"]


def test_ties_boundary_and_index_only():
    rng = np.random.default_rng(12)
    lengths = [1024, 1024, 2000, 900]
    num = float(np.power(np.float64(N_C), np.float64(ALPHA)))
    u_b = num / float(1024 * 1024)              # exact: u * n^2 == n_c^alpha, not kept whole
    u = np.array([u_b, np.nextafter(u_b, 0.0), 0.75, 0.999])
    keys = _keys(rng, int(np.sum(lengths)))
    keys[2048:4048] = 7                          # all keys equal: the first n_c positions
    res = _run(lengths, u, keys, seed=2)
    _check(res, lengths, u, keys)
    assert np.diff(res["out_offs"]).tolist()[:2] == [N_C, 1024]
    res = _run(lengths, u, keys, seed=2, with_values=False, with_ts=False)
    _check(res, lengths, u, keys, with_values=False, with_ts=False)


def test_lognormal_batch_of_sixteen_users():
    """The raw lengths of the 16-user lognormal workload (before sampling), d 512."""
    rng = np.random.default_rng(13)
    lengths = wl.draw_lengths("lognormal_1500_0.8_4096", 16, rng)
    u = rng.random(16)
    keys = _keys(rng, int(lengths.sum()))
    res = _run(lengths, u, keys, d=512, seed=3)
    _check(res, lengths, u, keys)


def test_empty_batch():
    res = _run([], np.zeros(0), np.zeros(0, np.uint32))
    assert res["out_offs"].tolist() == [0] and res["err"] == 0
    res = _run([0, 0], np.array([0.5, 0.5]), np.zeros(0, np.uint32))
    assert res["out_offs"].tolist() == [0, 0, 0] and res["err"] == 0


def test_too_long_and_bad_offsets_set_error_bits():
    rng = np.random.default_rng(14)
    # a sequence longer than the in-shared-memory sort that must be sampled: dropped, flagged
    lengths = [100, hstu.HSTU_SL_MAX_SAMPLED_LEN + 10, 900]
    u = np.array([0.5, 0.999, 0.999])
    keys = _keys(rng, int(np.sum(lengths)))
    res = _run(lengths, u, keys, d=64, seed=4)
    assert res["err"] == hstu.HSTU_DEVERR_SL_TOO_LONG
    ref_offs, ref_idx = oracle.stochastic_length(res["offs"], u, keys, N_C, ALPHA)
    kept = np.diff(res["out_offs"])
    assert kept[0] == 100 and kept[1] == 0 and kept[2] == np.diff(ref_offs)[2]
    # a decreasing offset table: the kernels clamp and flag it
    dev = "cuda:0"
    T, B = 100, 3
    offs = torch.tensor([0, 50, 30, 100], dtype=torch.int32, device=dev)
    u_d = torch.full((B,), 0.5, dtype=torch.float64, device=dev)
    keys_d = torch.zeros(T, dtype=torch.int32, device=dev)
    out_offs = torch.zeros(B + 1, dtype=torch.int32, device=dev)
    out_idx = torch.zeros(T, dtype=torch.int64, device=dev)
    scratch = torch.empty(hstu.hstu_stochastic_length_scratch_bytes(T, B), dtype=torch.uint8,
                          device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    hstu.hstu_stochastic_length(offs, B, T, u_d, keys_d, N_C, ALPHA, None, 0, None, out_offs,
                                out_idx, None, None, scratch, err, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(err.item()) & hstu.HSTU_DEVERR_OFFSETS
    o = out_offs.cpu().numpy()
    assert o[-1] <= T and np.all(np.diff(o) >= 0)
