"""fp64 CPU oracle of the jagged HSTU layer forward -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the package's smoke check and the benchmark's CPU
baseline leg may import this module.  The CUDA library never calls it and
shares no code with it: parity between the two is what the tests measure.

What it computes (one HSTU layer, per the pages; citations name the page and
its section/equation):

* Blog "Generative Recommendation 16: HSTU" (chenhuiyu.github.io), section
  "HSTU Layer 到底改了什么", equations (1)-(3):
      (1)  U, V, Q, K = Split(phi1(f1(X)))
      (2)  A(X)V = phi2(Q K^T + rab^{p,t}) V
      (3)  Y = f2(Norm(A(X)V) (.) U)
  with phi1 = phi2 = SiLU, and rab^{p,t} encoding relative position and the
  real time gap (same section, the sentence after the equations; ltzyclt blog
  on HSTU, section 4.1 note).
* Same blog, section "不对序列做 softmax": the SiLU is applied to every score
  on its own, with no normalisation along the sequence, and a LayerNorm
  follows the aggregation.
* Causal (autoregressive) setting over each user's time-ordered sequence
  (ltzyclt blog, section 3.2; aitrending "How Generative Recommenders Are
  Redefining RecSys at Scale", Technical Details: per-user sequences ordered
  by timestamp).  No attention crosses users: jagged batches are per-user
  sequences packed without padding (blog "Generative Recommendation 16",
  item 1 "Ragged/Jagged kernel").
* M-FALCON ranking mask: candidates attend to the cached history and not to
  each other; micro-batching only saves cost (ltzyclt blog, section 5.2; blog
  "Generative Recommendation 16", item 3 "M-FALCON").

Not on the pages, fixed by the layer configuration and taken as given here:
the 1/n_norm scale of the attention weights, the residual "+ X" after f2,
multi-head shapes (heads are contiguous column blocks of U, V, Q, K), the
bucket rules of rab (position: clamp(i - j, 0, pos_clamp); time:
floor(ln(1 + dt) / div) clamped to the last bucket) and the LayerNorm
epsilon.  Readings taken where the pages are silent:

* Split order is U, V, Q, K as contiguous chunks of width d.
* There is no 1/sqrt(head_dim) on the scores.
* Masked pairs contribute exactly 0 (not SiLU(-inf)).
* Both bias tables are shared by all heads.
* dt = t_query - t_key in integer seconds, clamped below at 0, natural log,
  computed in fp64.
* LayerNorm runs over the full d_model (all heads), biased variance, affine
  gamma/beta.
* f1 and f2 carry biases.
* M-FALCON: every candidate of a user sits at position n_h (the first
  position after that user's n_h history tokens); its self pair has relative
  position 0.  Results are therefore independent of the micro-batch split.

Every array here is float64 (int64 for indices).  This is a plain,
unblocked transcription: one dense masked n x n block per user and head.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Dict, Optional, Sequence

import numpy as np

CAUSAL = "causal"
MFALCON = "mfalcon"


@dataclass(frozen=True)
class OracleConfig:
    d_model: int
    num_heads: int
    head_dim: int
    pos_clamp: int
    time_buckets: int
    time_log_div: float
    n_norm: int          # > 0: fixed; <= 0: the longest sequence of the batch
    ln_eps: float = 1e-5
    mask: str = CAUSAL


def silu(x: np.ndarray) -> np.ndarray:
    """phi(x) = x * sigmoid(x) = x / (1 + e^{-x})."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def time_bucket(dt: np.ndarray, div: float, num_buckets: int) -> np.ndarray:
    """rab time index: floor(ln(1 + max(dt, 0)) / div), clamped to num_buckets - 1."""
    dt = np.maximum(np.asarray(dt, dtype=np.int64), 0).astype(np.float64)
    b = np.floor(np.log(1.0 + dt) / div)
    return np.minimum(b, num_buckets - 1).astype(np.int64)


def position_bucket(rel: np.ndarray, pos_clamp: int) -> np.ndarray:
    """rab position index: clamp(relative position, 0, pos_clamp)."""
    return np.clip(np.asarray(rel, dtype=np.int64), 0, pos_clamp)


def user_visibility(n: int, n_cand: int, mask: str, q_local: Optional[np.ndarray] = None):
    """Visibility and relative position for one user of length n.

    Returns (vis [m, n] bool, rel [m, n] int64) for the query rows ``q_local``
    (default: all n rows), where vis[r, j] says whether query q_local[r] may
    aggregate key j and rel[r, j] is the relative position used for the
    position bias.

    causal: key j is visible to query i iff j <= i; rel = i - j.
    mfalcon with n_h = n - n_cand history tokens: a history query i < n_h
    sees j <= i (rel = i - j); a candidate query i >= n_h sees every history
    key j < n_h (rel = n_h - j) and itself (rel = 0), never another candidate.
    """
    qi = np.arange(n) if q_local is None else np.asarray(q_local, dtype=np.int64)
    i = qi[:, None]
    j = np.arange(n)[None, :]
    if mask == CAUSAL or n_cand == 0:
        return (j <= i), (i - j)
    if mask != MFALCON:
        raise ValueError(mask)
    n_h = n - n_cand
    is_cand = i >= n_h
    vis = np.where(is_cand, (j < n_h) | (j == i), j <= i)
    rel = np.where(is_cand, np.where(j == i, 0, n_h - j), i - j)
    return vis, rel


def effective_n_norm(cfg: OracleConfig, lengths: Sequence[int]) -> float:
    if cfg.n_norm > 0:
        return float(cfg.n_norm)
    return float(max([int(n) for n in lengths] + [1]))


def f1_split(X: np.ndarray, W1: np.ndarray, b1: np.ndarray, d: int):
    """Equation (1): U, V, Q, K = Split(SiLU(X W1^T + b1))."""
    Z = silu(X @ W1.T + b1)
    return Z[:, 0:d], Z[:, d:2 * d], Z[:, 2 * d:3 * d], Z[:, 3 * d:4 * d]


def user_rab(ts_user: np.ndarray, q_local: np.ndarray, rel: np.ndarray, rab_pos: np.ndarray,
             rab_time: np.ndarray, cfg: OracleConfig):
    """rab^{p,t}[i, j] = rab_pos[pidx(i, j)] + rab_time[tidx(i, j)] for one user's query rows."""
    pidx = position_bucket(rel, cfg.pos_clamp)
    dt = ts_user[q_local][:, None] - ts_user[None, :]
    tidx = time_bucket(dt, cfg.time_log_div, cfg.time_buckets)
    return rab_pos[pidx] + rab_time[tidx], pidx, tidx


def pointwise_attention(Q, K, V, seq_offsets, timestamps, num_candidates,
                        rab_pos, rab_time, cfg: OracleConfig,
                        phi2: Callable[[np.ndarray], np.ndarray] = silu,
                        rows: Optional[np.ndarray] = None,
                        record: Optional[Dict] = None) -> np.ndarray:
    """Equation (2) with the jagged / causal / M-FALCON visibility.

    For each user b and head h, with local indices i, j of that user:
        a[i, j] = phi2(q_i . k_j + rab^{p,t}[i, j]) / n_norm   if visible
                = 0                                           otherwise
        O[i, head h] = sum_j a[i, j] v_j[head h]
    ``rows`` (optional, global row ids) limits which query rows are computed;
    all other output rows stay 0.  ``record`` (optional dict) receives the
    per-user (pidx, tidx, vis, a) arrays for inspection.
    """
    T = Q.shape[0]
    d, H, hd = cfg.d_model, cfg.num_heads, cfg.head_dim
    offs = np.asarray(seq_offsets, dtype=np.int64)
    lengths = offs[1:] - offs[:-1]
    nn = effective_n_norm(cfg, lengths)
    rab_pos = np.asarray(rab_pos, np.float64)
    rab_time = np.asarray(rab_time, np.float64)
    O = np.zeros((T, d), dtype=np.float64)
    want = None if rows is None else set(int(r) for r in rows)
    for b in range(len(lengths)):
        lo, hi = int(offs[b]), int(offs[b + 1])
        n = hi - lo
        if n == 0:
            continue
        n_c = int(num_candidates[b]) if (num_candidates is not None and cfg.mask == MFALCON) else 0
        q_local = np.arange(n)
        if want is not None:
            q_local = np.array([r - lo for r in range(lo, hi) if r in want], dtype=np.int64)
            if q_local.size == 0:
                continue
        vis, rel = user_visibility(n, n_c, cfg.mask, q_local)
        rab, pidx, tidx = user_rab(np.asarray(timestamps[lo:hi]), q_local, rel, rab_pos,
                                   rab_time, cfg)
        del rel
        for h in range(H):
            c0, c1 = h * hd, (h + 1) * hd
            s = Q[lo + q_local, c0:c1] @ K[lo:hi, c0:c1].T + rab
            a = np.where(vis, phi2(s) / nn, 0.0)
            O[lo + q_local, c0:c1] = a @ V[lo:hi, c0:c1]
            if record is not None:
                record.setdefault(b, {})[h] = a
        if record is not None:
            record.setdefault("buckets", {})[b] = (pidx, tidx, vis)
    return O


def layer_norm(O: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """Norm(.) of equation (3): per-row LayerNorm over d_model, biased variance."""
    mu = O.mean(axis=1, keepdims=True)
    var = ((O - mu) ** 2).mean(axis=1, keepdims=True)
    return (O - mu) / np.sqrt(var + eps) * gamma + beta


def hstu_layer(X, seq_offsets, timestamps, num_candidates, params, cfg: OracleConfig,
               phi2: Callable[[np.ndarray], np.ndarray] = silu,
               rows: Optional[np.ndarray] = None, record: Optional[Dict] = None):
    """One HSTU layer, equations (1)-(3) plus the residual: Y = f2(Norm(AV) (.) U) + X.

    ``params`` holds w1 [4d, d], b1 [4d], w2 [d, d], b2 [d], rab_pos, rab_time,
    ln_gamma, ln_beta (any float dtype; promoted to float64).  Returns a dict
    with Y and every intermediate (U, V, Q, K, O, N, G).  With ``rows`` only
    those output rows are meaningful (the rest of O, N, G, Y is not computed).
    """
    X = np.asarray(X, dtype=np.float64)
    p = {k: np.asarray(getattr(params, k) if not isinstance(params, dict) else params[k],
                       dtype=np.float64)
         for k in ("w1", "b1", "w2", "b2", "rab_pos", "rab_time", "ln_gamma", "ln_beta")}
    d = cfg.d_model
    U, V, Q, K = f1_split(X, p["w1"], p["b1"], d)
    O = pointwise_attention(Q, K, V, seq_offsets, timestamps, num_candidates,
                            p["rab_pos"], p["rab_time"], cfg, phi2=phi2, rows=rows,
                            record=record)
    if rows is None:
        N = layer_norm(O, p["ln_gamma"], p["ln_beta"], cfg.ln_eps)
        G = N * U
        Y = G @ p["w2"].T + p["b2"] + X
    else:
        rows = np.asarray(rows, dtype=np.int64)
        N = np.zeros_like(O)
        G = np.zeros_like(O)
        Y = np.zeros_like(X)
        N[rows] = layer_norm(O[rows], p["ln_gamma"], p["ln_beta"], cfg.ln_eps)
        G[rows] = N[rows] * U[rows]
        Y[rows] = G[rows] @ p["w2"].T + p["b2"] + X[rows]
    return {"U": U, "V": V, "Q": Q, "K": K, "O": O, "N": N, "G": G, "Y": Y}


def hstu_stack(X, seq_offsets, timestamps, num_candidates, layers, cfg: OracleConfig):
    """A stack of HSTU layers: the output of layer l is the input of layer l+1."""
    Y = np.asarray(X, dtype=np.float64)
    for params in layers:
        Y = hstu_layer(Y, seq_offsets, timestamps, num_candidates, params, cfg)["Y"]
    return Y


def visible_pairs(seq_offsets, num_candidates, mask: str) -> int:
    """Number of visible (query, key) pairs of a batch (for FLOP accounting)."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    total = 0
    for b in range(len(offs) - 1):
        n = int(offs[b + 1] - offs[b])
        n_c = int(num_candidates[b]) if (num_candidates is not None and mask == MFALCON) else 0
        n_h = n - n_c
        total += n_h * (n_h + 1) // 2 + n_c * (n_h + 1)
    return total
