"""CPU oracle of Stochastic Length sampling -- TEST INFRASTRUCTURE ONLY.

Only the test suite and the benchmark's CPU legs may import this module.  The
CUDA library never calls it and shares no code with it.

Stochastic Length (ltzyclt blog on HSTU, section 5.1; blog "Generative
Recommendation 16: HSTU", the three extra pieces, item 2): a user's sequence
of n actions is kept whole with probability N_c^alpha / n^2 (capped at 1);
otherwise a sub-sequence of it is sampled, which is what happens most of the
time for very long users -- alpha = 1.6 keeps length 4096 mostly at 776
actions -- and the sample is not simply the most recent actions.

Readings taken where the pages are silent:
* the sampled sub-sequence is a uniform subset of N_c positions drawn
  without replacement and kept in the original (time) order, so positions
  are recomputed on the kept sequence and timestamps travel with their
  actions;
* a sequence of n <= N_c actions is kept whole (no subset of N_c positions
  exists);
* the random numbers are inputs: one uniform u_b in [0, 1) per user, and the
  sequence is kept whole iff u_b * n^2 < N_c^alpha, evaluated in fp64 as
  written (n^2 exact, one rounding in the product; N_c^alpha from the C
  library's pow); one 32-bit key per action, and the subset is the N_c
  positions with the smallest (key, position) pairs -- a uniform subset when
  the keys are independent, uniform and distinct.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def keep_whole(n: int, u: float, n_c: int, alpha: float) -> bool:
    """Whether a length-n sequence with draw u is kept whole."""
    if n <= n_c:
        return True
    numerator = float(np.power(np.float64(n_c), np.float64(alpha)))
    return float(u) * float(n * n) < numerator


def stochastic_length(seq_offsets, user_uniform, token_keys, n_c: int,
                      alpha: float) -> Tuple[np.ndarray, np.ndarray]:
    """Stochastic Length over a jagged batch.

    seq_offsets: [B+1] offsets of the users' sequences in the packed token axis;
    user_uniform: [B] fp64 draws in [0, 1); token_keys: [T] uint32 draws.
    Returns (new_offsets [B+1], kept [T']) where kept lists, user after user
    and in time order, the global index of every action that survives."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    u = np.asarray(user_uniform, dtype=np.float64)
    keys = np.asarray(token_keys, dtype=np.uint64)
    B = offs.shape[0] - 1
    new_offsets = np.zeros(B + 1, dtype=np.int64)
    kept = []
    for b in range(B):
        lo, hi = int(offs[b]), int(offs[b + 1])
        n = hi - lo
        if keep_whole(n, u[b], n_c, alpha):
            chosen = np.arange(n, dtype=np.int64)
        else:
            # the n_c smallest (key, position) pairs, then back to time order
            by_key = np.lexsort((np.arange(n), keys[lo:hi]))
            chosen = np.sort(by_key[:n_c]).astype(np.int64)
        kept.append(lo + chosen)
        new_offsets[b + 1] = new_offsets[b] + chosen.shape[0]
    idx = np.concatenate(kept) if kept else np.zeros(0, dtype=np.int64)
    return new_offsets, idx.astype(np.int64)
