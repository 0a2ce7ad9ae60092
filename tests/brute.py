"""Element-by-element HSTU layer forward in pure Python scalars.

A second, independent transcription of the layer used to pin the vectorised
fp64 oracle on tiny inputs: every output element is one explicit sum, every
visibility and bias index one explicit branch.  It follows the same page
passages as the oracle (blog "Generative Recommendation 16: HSTU", section
"HSTU Layer 到底改了什么", equations (1)-(3); ltzyclt blog on HSTU, section
5.2 for the M-FALCON mask) but shares no code with it.
"""
import math


def _silu(x):
    if x < -700.0:
        return 0.0 * x
    return x / (1.0 + math.exp(-x))


def _pos_index(i, j, n, n_cand, mfalcon, pos_clamp):
    n_h = n - n_cand
    if mfalcon and i >= n_h:
        rel = 0 if i == j else n_h - j
    else:
        rel = i - j
    if rel < 0:
        return 0
    if rel > pos_clamp:
        return pos_clamp
    return rel


def _time_index(t_i, t_j, div, num_buckets):
    dt = t_i - t_j
    if dt < 0:
        dt = 0
    b = int(math.floor(math.log(1.0 + float(dt)) / div))
    return min(b, num_buckets - 1)


def _visible(i, j, n, n_cand, mfalcon):
    n_h = n - n_cand
    if mfalcon and i >= n_h:
        return j < n_h or j == i
    return j <= i


def brute_layer(X, seq_offsets, timestamps, num_candidates, p, d, H, hd, pos_clamp,
                time_buckets, div, n_norm, eps, mfalcon):
    """Returns dict of python lists: U, V, Q, K, O, Y (row-major nested lists)."""
    T = len(X)
    w1, b1, w2, b2 = p["w1"], p["b1"], p["w2"], p["b2"]
    rp, rt, g, be = p["rab_pos"], p["rab_time"], p["ln_gamma"], p["ln_beta"]
    Z = [[0.0] * (4 * d) for _ in range(T)]
    for t in range(T):
        for o in range(4 * d):
            acc = float(b1[o])
            for k in range(d):
                acc += float(X[t][k]) * float(w1[o][k])
            Z[t][o] = _silu(acc)
    U = [row[0:d] for row in Z]
    V = [row[d:2 * d] for row in Z]
    Q = [row[2 * d:3 * d] for row in Z]
    K = [row[3 * d:4 * d] for row in Z]
    lengths = [int(seq_offsets[b + 1]) - int(seq_offsets[b]) for b in range(len(seq_offsets) - 1)]
    nn = float(n_norm) if n_norm > 0 else float(max(lengths + [1]))
    O = [[0.0] * d for _ in range(T)]
    for b in range(len(lengths)):
        lo = int(seq_offsets[b])
        n = lengths[b]
        nc = int(num_candidates[b]) if mfalcon else 0
        for i in range(n):
            for h in range(H):
                for c in range(hd):
                    acc = 0.0
                    for j in range(n):
                        if not _visible(i, j, n, nc, mfalcon):
                            continue
                        s = 0.0
                        for k in range(hd):
                            s += Q[lo + i][h * hd + k] * K[lo + j][h * hd + k]
                        s += float(rp[_pos_index(i, j, n, nc, mfalcon, pos_clamp)])
                        s += float(rt[_time_index(int(timestamps[lo + i]), int(timestamps[lo + j]),
                                                  div, time_buckets)])
                        acc += _silu(s) / nn * V[lo + j][h * hd + c]
                    O[lo + i][h * hd + c] = acc
    Y = [[0.0] * d for _ in range(T)]
    for t in range(T):
        mu = sum(O[t]) / d
        var = sum((o - mu) ** 2 for o in O[t]) / d
        Nrow = [(O[t][c] - mu) / math.sqrt(var + eps) * float(g[c]) + float(be[c]) for c in range(d)]
        Grow = [Nrow[c] * U[t][c] for c in range(d)]
        for o in range(d):
            acc = float(b2[o]) + float(X[t][o])
            for c in range(d):
                acc += Grow[c] * float(w2[o][c])
            Y[t][o] = acc
    return {"U": U, "V": V, "Q": Q, "K": K, "O": O, "Y": Y}
