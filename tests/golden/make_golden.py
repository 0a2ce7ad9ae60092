"""Writes the tiny regression fixtures under tests/golden/ from the fp64 oracle.

Inputs are closed-form tiny tensors defined here; expected values come only
from oracle/.  Re-run after a deliberate, justified change to the oracle:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import OracleConfig, hstu_layer  # noqa: E402


def tiny_inputs(mask):
    d, H = 4, 2
    if mask == "causal":
        lengths, ncand = [3, 0, 4], [0, 0, 0]
    else:
        lengths, ncand = [5, 2], [2, 1]
    T = sum(lengths)
    t = np.arange(T, dtype=np.float64)
    X = np.sin(0.7 * t[:, None] + np.arange(d)[None, :]) * 0.9
    W1 = np.cos(0.31 * np.arange(4 * d)[:, None] - 0.53 * np.arange(d)[None, :]) * 0.6
    b1 = 0.05 * np.arange(4 * d) - 0.3
    W2 = np.sin(0.41 * np.arange(d)[:, None] + 0.29 * np.arange(d)[None, :]) * 0.5
    b2 = np.linspace(-0.2, 0.2, d)
    rab_pos = np.linspace(-0.5, 0.5, 9)
    rab_time = 0.1 * np.cos(np.arange(12))
    gamma = 1.0 + 0.1 * np.arange(d)
    beta = -0.05 * np.arange(d)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    ts = []
    for n in lengths:
        ts += [1000 + 7 * k * k for k in range(n)]
    p = dict(w1=W1, b1=b1, w2=W2, b2=b2, rab_pos=rab_pos, rab_time=rab_time,
             ln_gamma=gamma, ln_beta=beta)
    cfg = OracleConfig(d_model=d, num_heads=H, head_dim=d // H, pos_clamp=8, time_buckets=12,
                       time_log_div=0.301, n_norm=0 if mask == "causal" else 4, ln_eps=1e-5,
                       mask=mask)
    return X, offs, np.array(ts, np.int64), np.array(ncand, np.int32), p, cfg


def main():
    for mask in ("causal", "mfalcon"):
        X, offs, ts, nc, p, cfg = tiny_inputs(mask)
        out = hstu_layer(X, offs, ts, nc, p, cfg)
        doc = {"note": "regression fixture written by tests/golden/make_golden.py from oracle/",
               "mask": mask, "O": out["O"].tolist(), "Y": out["Y"].tolist()}
        with open(os.path.join(HERE, f"tiny_layer_{mask}.json"), "w") as f:
            json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
