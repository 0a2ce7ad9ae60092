"""Checks of the seeded input generators (shapes, laws, Stochastic Length)."""
import json
import os

import numpy as np
import pytest
import torch

from jagged_pointwise_attention_hstu_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_zipf_truncated_mean():
    rng = np.random.default_rng(0)
    n = wl.draw_lengths("zipf_1.2_32_1024", 200_000, rng)
    assert n.min() >= 32 and n.max() <= 1024
    k = np.arange(32, 1025, dtype=np.float64)
    p = k ** -1.2
    exact_mean = float((k * p).sum() / p.sum())
    assert abs(exact_mean - 239.0) < 1.0
    assert abs(n.mean() - exact_mean) < 3.0


def test_stochastic_length_matches_page_numbers():
    """alpha = 1.6 maps length 4096 mostly to 776 (ltzyclt blog on HSTU, section 5.1;
    blog "Generative Recommendation 16", item 2 "Stochastic Length")."""
    with open(os.path.join(GOLDEN, "stochastic_length.json")) as f:
        g = json.load(f)
    assert g["n"] ** (g["alpha"] / 2) == pytest.approx(g["kept"], abs=0.5)
    p = float(wl.sl_keep_full_probability(np.array([g["n"]]))[0])
    assert p == pytest.approx(g["kept"] ** g["alpha"] / g["n"] ** 2)
    assert p < 0.01                       # "mostly" truncated
    rng = np.random.default_rng(5)
    sizes = [wl.stochastic_length_positions(4096, rng).shape[0] for _ in range(4000)]
    frac_full = np.mean(np.array(sizes) == 4096)
    assert abs(frac_full - p) < 0.004
    assert set(sizes) <= {4096, 776}


def test_stochastic_length_keep_probability_monte_carlo():
    rng = np.random.default_rng(9)
    for n in (900, 1500, 2500):
        p = float(wl.sl_keep_full_probability(np.array([n]))[0])
        kept = [wl.stochastic_length_positions(n, rng) for _ in range(3000)]
        frac = np.mean([k.shape[0] == n for k in kept])
        assert abs(frac - p) < 4 * np.sqrt(p * (1 - p) / 3000) + 1e-3
        for k in kept[:50]:
            assert np.all(np.diff(k) > 0) and k[0] >= 0 and k[-1] < n
    # never subsampled below N_c
    assert wl.stochastic_length_positions(500, rng).shape[0] == 500


@pytest.mark.parametrize("idx", [0, 1, 2, 4])
def test_batches_are_well_formed(idx):
    w = wl.WORKLOADS[idx]
    b = wl.make_batch(w)
    offs = b.seq_offsets.astype(np.int64)
    assert offs[0] == 0 and np.all(np.diff(offs) >= 0) and offs[-1] == b.total_tokens
    assert b.x.shape == (b.total_tokens, w.d_model) and b.x.dtype == np.float32
    for u in range(b.num_users):
        ts = b.timestamps[offs[u]:offs[u + 1]]
        assert np.all(np.diff(ts) >= 0)
        if w.mask == "mfalcon":
            nh = (offs[u + 1] - offs[u]) - b.num_candidates[u]
            assert np.all(ts[nh:] == ts[nh - 1])
    assert len(b.layers) == w.num_layers
    assert b.layers[0].rab_pos.shape == (w.pos_buckets,)
    # same seed, same bytes
    b2 = wl.make_batch(w)
    assert np.array_equal(b.x, b2.x) and np.array_equal(b.timestamps, b2.timestamps)


def test_stack_prefix_batch_holds_leading_rows():
    w = wl.WORKLOADS[3]
    full = wl.make_batch(w, num_layers=1, num_users=2)
    pre = wl.make_batch(w, num_layers=1, num_users=2, max_len=256)
    offs = full.seq_offsets
    rows = np.concatenate([np.arange(offs[u], offs[u] + 256) for u in range(2)])
    assert np.array_equal(pre.x, full.x[rows])
    assert np.array_equal(pre.timestamps, full.timestamps[rows])
    assert np.array_equal(pre.layers[0].w1, full.layers[0].w1)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    a = (rng.normal(0, 3, size=10000) * 10.0 ** rng.integers(-6, 6, size=10000)).astype(np.float32)
    ours = wl.round_to_storage(a, "bf16")
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours, ref)
    bits = wl.to_bf16_bits(a)
    assert np.array_equal(bits, torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy()
                          .view(np.uint16))
