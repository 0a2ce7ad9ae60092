"""Pins of the backward oracle against things other than itself.

* finite differences of the (already pinned) forward oracle: for every input
  and parameter, the directional derivative of sum(dY * Y) along random
  directions, by central differences in fp64;
* torch autograd in float64 through a forward written here from the layer's
  equations with torch's own LayerNorm -- a different mechanism for every
  derivative;
* closed forms: with W2 = 0 no gradient reaches anything before f2 and
  dX = dY exactly; dW2 = dY^T G and db2 = sum(dY) always;
* a planted slip (SiLU's derivative replaced by the sigmoid) fails the
  finite-difference pin.
Small shapes (d 8, two heads) with strong weights and bias tables so that
every term matters; causal and M-FALCON masks, fixed and per-batch n_norm.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import hstu_backward as hb

from helpers import oracle_cfg

KEYS = ("w1", "b1", "w2", "b2", "rab_pos", "rab_time", "ln_gamma", "ln_beta")
D, H, CLAMP, NB, DIV = 8, 2, 3, 16, 0.301


def _case(seed, mask, n_norm):
    rng = np.random.default_rng(seed)
    lengths = [4, 0, 6, 1, 3]
    ncand = [0, 0, 2, 1, 1] if mask == "mfalcon" else [0] * 5
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offs[-1])
    ts = np.concatenate([np.sort(rng.integers(0, 5000, size=n)) for n in lengths]).astype(np.int64)
    p = {"w1": rng.normal(0, 0.5, (4 * D, D)), "b1": rng.normal(0, 0.3, 4 * D),
         "w2": rng.normal(0, 0.5, (D, D)), "b2": rng.normal(0, 0.3, D),
         "rab_pos": rng.normal(0, 1.0, CLAMP + 1), "rab_time": rng.normal(0, 1.0, NB),
         "ln_gamma": rng.normal(1, 0.3, D), "ln_beta": rng.normal(0, 0.3, D)}
    X = rng.normal(0, 1, (T, D))
    dY = rng.normal(0, 1, (T, D))
    cfg = oracle_cfg(D, H, pos_clamp=CLAMP, time_buckets=NB, div=DIV, n_norm=n_norm, mask=mask)
    return X, offs, ts, np.array(ncand), p, cfg, dY


def _loss(X, offs, ts, ncand, p, cfg, dY):
    return float(np.sum(dY * oracle.hstu_layer(X, offs, ts, ncand, p, cfg)["Y"]))


@pytest.mark.parametrize("mask,n_norm", [("causal", 0), ("causal", 5), ("mfalcon", 7)])
def test_finite_differences(mask, n_norm):
    X, offs, ts, ncand, p, cfg, dY = _case(1, mask, n_norm)
    g = hb.hstu_layer_backward(X, offs, ts, ncand, p, cfg, dY)
    rng = np.random.default_rng(2)
    eps = 1e-6
    for key in KEYS + ("X",):
        base = X if key == "X" else p[key]
        for _ in range(3):
            v = rng.normal(size=base.shape)
            plus = base + eps * v
            minus = base - eps * v
            if key == "X":
                fd = (_loss(plus, offs, ts, ncand, p, cfg, dY)
                      - _loss(minus, offs, ts, ncand, p, cfg, dY)) / (2 * eps)
            else:
                fd = (_loss(X, offs, ts, ncand, {**p, key: plus}, cfg, dY)
                      - _loss(X, offs, ts, ncand, {**p, key: minus}, cfg, dY)) / (2 * eps)
            an = float(np.sum(g[key] * v))
            assert abs(fd - an) <= 1e-6 * (abs(an) + 1.0), (key, fd, an)


def _torch_layer(X, offs, ts, ncand, p, mask, n_norm, eps):
    """The layer in torch float64, written from equations (1)-(3) plus the residual."""
    w1, b1, w2, b2 = p["w1"], p["b1"], p["w2"], p["b2"]
    H1 = X @ w1.T + b1
    Z = H1 * torch.sigmoid(H1)
    U, V, Q, K = Z[:, :D], Z[:, D:2 * D], Z[:, 2 * D:3 * D], Z[:, 3 * D:]
    lengths = [int(offs[b + 1] - offs[b]) for b in range(len(offs) - 1)]
    nn = float(n_norm if n_norm > 0 else max(lengths + [1]))
    hd = D // H
    pieces = []
    for b, n in enumerate(lengths):
        if n == 0:
            continue
        lo = int(offs[b])
        vis = np.zeros((n, n), bool)
        rel = np.zeros((n, n), np.int64)
        n_h = n - int(ncand[b]) if mask == "mfalcon" else n
        for i in range(n):
            for j in range(n):
                if i < n_h:
                    vis[i, j] = j <= i
                    rel[i, j] = i - j
                else:                      # a candidate: the history and itself
                    vis[i, j] = j < n_h or j == i
                    rel[i, j] = 0 if j == i else n_h - j
        pidx = np.minimum(np.maximum(rel, 0), CLAMP)
        dt = np.maximum(ts[lo:lo + n][:, None] - ts[lo:lo + n][None, :], 0).astype(np.float64)
        tidx = np.minimum(np.floor(np.log1p(dt) / DIV), NB - 1).astype(np.int64)
        rab = p["rab_pos"][torch.from_numpy(pidx)] + p["rab_time"][torch.from_numpy(tidx)]
        m = torch.from_numpy(vis)
        heads = []
        for h in range(H):
            c = slice(h * hd, (h + 1) * hd)
            s = Q[lo:lo + n, c] @ K[lo:lo + n, c].T + rab
            a = torch.where(m, s * torch.sigmoid(s) / nn, torch.zeros_like(s))
            heads.append(a @ V[lo:lo + n, c])
        pieces.append(torch.cat(heads, dim=1))
    O = torch.cat(pieces, dim=0)
    N = torch.nn.functional.layer_norm(O, (D,), p["ln_gamma"], p["ln_beta"], eps)
    return (N * U) @ w2.T + b2 + X


@pytest.mark.parametrize("mask,n_norm", [("causal", 0), ("mfalcon", 7)])
def test_torch_autograd(mask, n_norm):
    X, offs, ts, ncand, p, cfg, dY = _case(3, mask, n_norm)
    g = hb.hstu_layer_backward(X, offs, ts, ncand, p, cfg, dY)
    tp = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in p.items()}
    tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    Y = _torch_layer(tX, offs, ts, ncand, tp, mask, n_norm, cfg.ln_eps)
    assert np.allclose(Y.detach().numpy(), oracle.hstu_layer(X, offs, ts, ncand, p, cfg)["Y"],
                       atol=1e-12)
    (Y * torch.from_numpy(dY)).sum().backward()
    for k in KEYS:
        assert np.allclose(g[k], tp[k].grad.numpy(), rtol=1e-10, atol=1e-11), k
    assert np.allclose(g["X"], tX.grad.numpy(), rtol=1e-10, atol=1e-11)


def test_closed_forms():
    X, offs, ts, ncand, p, cfg, dY = _case(4, "causal", 0)
    g = hb.hstu_layer_backward(X, offs, ts, ncand, p, cfg, dY)
    G = oracle.hstu_layer(X, offs, ts, ncand, p, cfg)["G"]
    assert np.allclose(g["w2"], dY.T @ G, rtol=1e-13, atol=1e-13)
    assert np.array_equal(g["b2"], dY.sum(axis=0))
    q = dict(p, w2=np.zeros_like(p["w2"]))
    g0 = hb.hstu_layer_backward(X, offs, ts, ncand, q, cfg, dY)
    assert np.array_equal(g0["X"], dY)
    for k in ("w1", "b1", "rab_pos", "rab_time", "ln_gamma", "ln_beta"):
        assert not np.any(g0[k]), k


def test_planted_slip_fails_the_finite_difference_pin(monkeypatch):
    X, offs, ts, ncand, p, cfg, dY = _case(5, "causal", 0)
    monkeypatch.setattr(hb, "silu_grad", hb.sigmoid)
    g = hb.hstu_layer_backward(X, offs, ts, ncand, p, cfg, dY)
    v = np.random.default_rng(6).normal(size=p["w1"].shape)
    eps = 1e-6
    fd = (_loss(X, offs, ts, ncand, {**p, "w1": p["w1"] + eps * v}, cfg, dY)
          - _loss(X, offs, ts, ncand, {**p, "w1": p["w1"] - eps * v}, cfg, dY)) / (2 * eps)
    assert abs(fd - float(np.sum(g["w1"] * v))) > 1e-3 * (abs(fd) + 1.0)
