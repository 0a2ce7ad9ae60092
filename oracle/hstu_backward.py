"""fp64 CPU oracle of the HSTU layer BACKWARD -- TEST INFRASTRUCTURE ONLY.

Only the test suite may import this module; the CUDA library shares no code
with it.

The pages describe training -- the speed ratios quoted "in training" (atlas
summary, key results; ltzyclt blog on HSTU, section 6.1) and the activation
memory of 14d per layer (ltzyclt blog, section 4.2; blog "Generative
Recommendation 16", section "用门控代替独立 FFN") -- but print no gradient.
The backward here is the exact derivative of the forward that
``hstu_oracle.hstu_layer`` computes (equations (1)-(3) of blog "Generative
Recommendation 16", section "HSTU Layer 到底改了什么", plus the residual),
taken by the chain rule one step at a time in the reverse order of the
forward: the residual and f2, the gate, the LayerNorm, the pointwise
attention (per user and head, over the same visible pairs), then SiLU and f1.
Bucket indices are integers and carry no gradient; the gradients of the two
bias tables sum the score gradients over every (query, key, head) that reads
each entry, since the tables are shared by all heads.

Every array is float64.  Plain, unblocked, one dense masked block per user
and head, like the forward.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from .hstu_oracle import (MFALCON, OracleConfig, effective_n_norm, pointwise_attention, silu,
                          user_rab, user_visibility)


def sigmoid(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def silu_grad(x: np.ndarray) -> np.ndarray:
    """d/dx [x sigmoid(x)] = sigmoid(x) (1 + x (1 - sigmoid(x)))."""
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


def _params(params) -> Dict[str, np.ndarray]:
    return {k: np.asarray(getattr(params, k) if not isinstance(params, dict) else params[k],
                          dtype=np.float64)
            for k in ("w1", "b1", "w2", "b2", "rab_pos", "rab_time", "ln_gamma", "ln_beta")}


def pointwise_attention_backward(Q, K, V, dO, seq_offsets, timestamps, num_candidates,
                                 rab_pos, rab_time, cfg: OracleConfig):
    """Gradients of sum(dO * O) for O = pointwise_attention(Q, K, V, ...):
    returns (dQ, dK, dV, d_rab_pos, d_rab_time).  Per user and head, with
    s = q.k + rab and a = vis * SiLU(s) / n_norm:
        dV = a^T dO,  dA = dO V^T,  dS = vis * dA * SiLU'(s) / n_norm,
        dQ = dS K,    dK = dS^T Q,
    and each bias entry collects dS of every visible (query, key, head) that
    reads it."""
    Q, K, V, dO = (np.asarray(x, dtype=np.float64) for x in (Q, K, V, dO))
    rab_pos = np.asarray(rab_pos, dtype=np.float64)
    rab_time = np.asarray(rab_time, dtype=np.float64)
    H, hd = cfg.num_heads, cfg.head_dim
    offs = np.asarray(seq_offsets, dtype=np.int64)
    lengths = offs[1:] - offs[:-1]
    nn = effective_n_norm(cfg, lengths)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    d_pos = np.zeros_like(rab_pos)
    d_time = np.zeros_like(rab_time)
    for b in range(len(lengths)):
        lo, hi = int(offs[b]), int(offs[b + 1])
        n = hi - lo
        if n == 0:
            continue
        n_c = int(num_candidates[b]) if (num_candidates is not None and cfg.mask == MFALCON) else 0
        q_local = np.arange(n)
        vis, rel = user_visibility(n, n_c, cfg.mask, q_local)
        rab, pidx, tidx = user_rab(np.asarray(timestamps[lo:hi]), q_local, rel, rab_pos,
                                   rab_time, cfg)
        d_rab = np.zeros(vis.shape)
        for h in range(H):
            c = slice(h * hd, (h + 1) * hd)
            s = Q[lo:hi, c] @ K[lo:hi, c].T + rab
            a = np.where(vis, silu(s) / nn, 0.0)
            dV[lo:hi, c] += a.T @ dO[lo:hi, c]
            da = dO[lo:hi, c] @ V[lo:hi, c].T
            ds = np.where(vis, da * silu_grad(s) / nn, 0.0)
            dQ[lo:hi, c] += ds @ K[lo:hi, c]
            dK[lo:hi, c] += ds.T @ Q[lo:hi, c]
            d_rab += ds
        np.add.at(d_pos, pidx[vis], d_rab[vis])
        np.add.at(d_time, tidx[vis], d_rab[vis])
    return dQ, dK, dV, d_pos, d_time


def hstu_layer_backward(X, seq_offsets, timestamps, num_candidates, params, cfg: OracleConfig,
                        dY) -> Dict[str, np.ndarray]:
    """Gradients of sum(dY * Y) for Y = hstu_layer(X, ...)["Y"].

    Returns dX and the gradient of every parameter, keyed like ``params``:
    w1, b1, w2, b2, rab_pos, rab_time, ln_gamma, ln_beta (and "X")."""
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    p = _params(params)
    d = cfg.d_model

    # ---- forward, keeping what the backward reads
    H1 = X @ p["w1"].T + p["b1"]                       # equation (1), before phi1
    Z = silu(H1)
    U, V, Q, K = Z[:, :d], Z[:, d:2 * d], Z[:, 2 * d:3 * d], Z[:, 3 * d:]
    O = pointwise_attention(Q, K, V, seq_offsets, timestamps, num_candidates, p["rab_pos"],
                            p["rab_time"], cfg)
    mu = O.mean(axis=1, keepdims=True)
    var = ((O - mu) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + cfg.ln_eps)
    Ohat = (O - mu) * rstd
    N = Ohat * p["ln_gamma"] + p["ln_beta"]
    G = N * U

    # ---- equation (3) and the residual: Y = G W2^T + b2 + X
    g = {}
    dX = dY.copy()
    g["w2"] = dY.T @ G
    g["b2"] = dY.sum(axis=0)
    dG = dY @ p["w2"]
    # gate: G = N (.) U
    dN = dG * U
    dU = dG * N
    # LayerNorm: N = Ohat gamma + beta, Ohat = (O - mu) rstd, over each row
    g["ln_gamma"] = (dN * Ohat).sum(axis=0)
    g["ln_beta"] = dN.sum(axis=0)
    dOhat = dN * p["ln_gamma"]
    dO = rstd * (dOhat - dOhat.mean(axis=1, keepdims=True)
                 - Ohat * (dOhat * Ohat).mean(axis=1, keepdims=True))

    # ---- equation (2): O = a V with a = vis * SiLU(Q K^T + rab) / n_norm
    dQ, dK, dV, g["rab_pos"], g["rab_time"] = pointwise_attention_backward(
        Q, K, V, dO, seq_offsets, timestamps, num_candidates, p["rab_pos"], p["rab_time"], cfg)

    # ---- equation (1): Z = SiLU(X W1^T + b1), split U | V | Q | K
    dZ = np.concatenate([dU, dV, dQ, dK], axis=1)
    dH1 = dZ * silu_grad(H1)
    g["w1"] = dH1.T @ X
    g["b1"] = dH1.sum(axis=0)
    dX += dH1 @ p["w1"]
    g["X"] = dX
    return g
