"""Pins of the Stochastic Length oracle against things other than itself.

The rule (ltzyclt blog on HSTU, section 5.1; blog "Generative Recommendation
16: HSTU", item 2 "Stochastic Length"): keep a length-n sequence whole with
probability N_c^alpha / n^2, else sample a sub-sequence; alpha = 1.6 keeps
length 4096 mostly at 776 actions.  Pins:
* the page's worked numbers (tests/golden/stochastic_length.json) and the
  keep rate by Monte Carlo against the closed form min(1, N_c^alpha / n^2);
* the subset by an independent formulation: position i survives iff fewer
  than N_c positions precede it in (key, position) order, counted pair by
  pair, and its inclusion frequency is N_c / n for every position;
* the decision boundary exactly: with n^2 a power of two, u = N_c^alpha / n^2
  is exact, so u * n^2 equals N_c^alpha and the sequence is NOT kept whole
  (strict inequality), while the next double below keeps it;
* jagged structure: offsets are the running sums, indices stay inside their
  user and increase, users are independent.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
N_C, ALPHA = 776, 1.6


def _one(n, u, keys, n_c=N_C, alpha=ALPHA):
    offs, idx = oracle.stochastic_length(np.array([0, n]), np.array([u]),
                                         np.asarray(keys, np.uint32), n_c, alpha)
    assert offs[0] == 0 and offs[1] == idx.shape[0]
    return idx


def test_short_sequences_are_kept_whole():
    rng = np.random.default_rng(1)
    for n in (0, 1, 5, 775, 776):
        keys = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
        assert np.array_equal(_one(n, 0.999999, keys), np.arange(n))


def test_page_numbers_and_keep_rate():
    with open(os.path.join(GOLDEN, "stochastic_length.json")) as f:
        g = json.load(f)
    rng = np.random.default_rng(2)
    for n in (900, 1500, 2500, g["n"]):
        p = min(1.0, g["kept"] ** g["alpha"] / n ** 2)
        trials = 4000
        whole = 0
        for _ in range(trials):
            keys = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
            k = _one(n, rng.random(), keys, g["kept"], g["alpha"]).shape[0]
            assert k in (n, g["kept"])
            whole += k == n
        assert abs(whole / trials - p) < 4 * np.sqrt(p * (1 - p) / trials) + 1e-3
    # "mostly" 776 for 4096
    assert g["kept"] ** g["alpha"] / g["n"] ** 2 < 0.01


def test_subset_by_counting_ranks():
    rng = np.random.default_rng(3)
    for trial in range(60):
        n = int(rng.integers(6, 40))
        n_c = int(rng.integers(1, n))
        keys = rng.integers(0, 8, size=n).astype(np.uint32)      # many ties
        idx = _one(n, 0.9999999, keys, n_c, 10.0 if trial % 2 else 0.5)
        if idx.shape[0] == n:      # kept whole: only possible when u n^2 < n_c^alpha
            assert 0.9999999 * n * n < n_c ** (10.0 if trial % 2 else 0.5)
            continue
        expect = []
        for i in range(n):
            ahead = sum(1 for j in range(n) if (keys[j], j) < (keys[i], i))
            if ahead < n_c:
                expect.append(i)
        assert idx.tolist() == expect


def test_subset_is_uniform():
    rng = np.random.default_rng(4)
    n, n_c, trials = 40, 10, 4000
    counts = np.zeros(n)
    for _ in range(trials):
        keys = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
        idx = _one(n, 0.999, keys, n_c, 1.0)          # 10 / 1600 < 0.999: subsampled
        assert idx.shape[0] == n_c and np.all(np.diff(idx) > 0)
        counts[idx] += 1
    p = n_c / n
    assert np.all(np.abs(counts / trials - p) < 4 * np.sqrt(p * (1 - p) / trials))


def test_decision_boundary_is_strict():
    n = 1024                                        # n^2 = 2^20: the division is exact
    num = float(np.power(np.float64(N_C), np.float64(ALPHA)))
    u = num / float(n * n)
    assert u * float(n * n) == num
    keys = np.arange(n, dtype=np.uint32)[::-1].copy()
    assert _one(n, u, keys).shape[0] == N_C
    assert _one(n, np.nextafter(u, 0.0), keys).shape[0] == n
    assert not oracle.keep_whole(n, u, N_C, ALPHA)
    assert oracle.keep_whole(n, np.nextafter(u, 0.0), N_C, ALPHA)


def test_jagged_structure_and_user_independence():
    rng = np.random.default_rng(5)
    lengths = np.array([0, 3000, 1, 0, 800, 5000, 776, 777])
    offs = np.concatenate([[0], np.cumsum(lengths)])
    T = int(offs[-1])
    u = rng.random(lengths.shape[0])
    keys = rng.integers(0, 2 ** 32, size=T, dtype=np.uint64).astype(np.uint32)
    new_offs, idx = oracle.stochastic_length(offs, u, keys, N_C, ALPHA)
    assert new_offs[0] == 0 and new_offs[-1] == idx.shape[0]
    for b in range(lengths.shape[0]):
        part = idx[new_offs[b]:new_offs[b + 1]]
        assert np.all((part >= offs[b]) & (part < offs[b + 1]))
        assert np.all(np.diff(part) > 0)
        # each user alone gives the same kept positions
        alone = _one(int(lengths[b]), u[b], keys[offs[b]:offs[b + 1]])
        assert np.array_equal(part - offs[b], alone)
