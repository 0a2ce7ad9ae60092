"""Pins of the fp64 oracle against things other than itself.

* brute force: a scalar, element-by-element transcription (tests/brute.py);
* library routines: SiLU, LayerNorm and Linear from torch in float64;
* closed forms: special weights for which equations (1)-(3) of blog
  "Generative Recommendation 16: HSTU" (section "HSTU Layer 到底改了什么")
  reduce to a formula that needs no attention loop;
* exact mathematics: the time-bucket rule evaluated with 60-digit decimals;
* invariants stated by the pages: causality (ltzyclt blog, section 3.2), no
  cross-user attention on jagged batches ("Ragged/Jagged kernel" item), and
  the M-FALCON property that candidates do not see each other and that
  micro-batching only saves cost (ltzyclt blog, section 5.2).

Each pin is chosen so that a plausible slip in the oracle -- a dropped bias
term, a transposed product, a wrong split order, an off-by-one in the mask or
in a bucket index, a softmax sneaking in -- fails at least one of them; the
mutation tests at the end plant such slips and check that.
"""
import decimal
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import hstu_oracle as ho
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from brute import brute_layer
from helpers import oracle_cfg, params_dict, max_abs


def _run_both(batch, cfg):
    p = params_dict(batch.layers[0])
    X = batch.x.astype(np.float64)
    o = oracle.hstu_layer(X, batch.seq_offsets, batch.timestamps, batch.num_candidates, p, cfg)
    b = brute_layer(X.tolist(), batch.seq_offsets, batch.timestamps, batch.num_candidates,
                    {k: v.tolist() for k, v in p.items()}, cfg.d_model, cfg.num_heads,
                    cfg.head_dim, cfg.pos_clamp, cfg.time_buckets, cfg.time_log_div,
                    cfg.n_norm, cfg.ln_eps, cfg.mask == "mfalcon")
    return o, b


@pytest.mark.parametrize("lengths,ncand,mask,n_norm", [
    ([5, 0, 9, 1], None, "causal", 0),
    ([7, 3, 12], None, "causal", 16),
    ([9, 6, 0, 11], [4, 0, 0, 5], "mfalcon", 12),
    ([4, 8], [4, 3], "mfalcon", 0),          # a user made only of candidates
])
def test_oracle_matches_brute_force(lengths, ncand, mask, n_norm):
    d, H = 8, 2
    batch = wl.make_custom_batch(lengths, d, H, seed=len(lengths) + (n_norm or 0),
                                 num_candidates=ncand, pos_buckets=9, time_buckets=20,
                                 weight_scale=0.7, rab_scale=1.5, random_affine=True,
                                 timestamp_gap=5.0)
    cfg = oracle_cfg(d, H, pos_clamp=8, time_buckets=20, n_norm=n_norm, mask=mask)
    o, b = _run_both(batch, cfg)
    for key in ("U", "V", "Q", "K", "O", "Y"):
        assert max_abs(o[key], b[key]) <= 1e-12 * max(1.0, np.abs(o[key]).max()), key


def test_library_routines_silu_layernorm_linear():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 4, size=(64, 32))
    assert max_abs(oracle.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy()) < 1e-15
    g = rng.normal(1, 0.2, size=32)
    b = rng.normal(0, 0.2, size=32)
    ln_t = torch.nn.functional.layer_norm(torch.from_numpy(x), (32,), torch.from_numpy(g),
                                          torch.from_numpy(b), eps=1e-5).numpy()
    assert max_abs(oracle.layer_norm(x, g, b, 1e-5), ln_t) < 1e-12
    W1 = rng.normal(0, 0.3, size=(4 * 32, 32))
    b1 = rng.normal(0, 0.3, size=4 * 32)
    lin = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(W1), torch.from_numpy(b1))
    Z = torch.nn.functional.silu(lin).numpy()
    U, V, Q, K = oracle.f1_split(x, W1, b1, 32)
    assert max_abs(np.concatenate([U, V, Q, K], axis=1), Z) < 1e-12
    # the split order is U, V, Q, K: the first d outputs are the gate U
    assert max_abs(U, Z[:, :32]) < 1e-12 and max_abs(K, Z[:, 96:]) < 1e-12


# ---------------------------------------------------------------- closed forms

def _tiny(lengths, ncand=None, mask="causal", d=16, H=2, seed=3, n_norm=0):
    batch = wl.make_custom_batch(lengths, d, H, seed=seed, num_candidates=ncand,
                                 weight_scale=0.3, rab_scale=0.8, random_affine=True)
    cfg = oracle_cfg(d, H, n_norm=n_norm, mask=mask)
    return batch, cfg, params_dict(batch.layers[0])


def test_closed_form_zero_f2_gives_residual_plus_bias():
    batch, cfg, p = _tiny([6, 3, 10])
    p["w2"][:] = 0.0
    out = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, None, p, cfg)
    assert max_abs(out["Y"], batch.x.astype(np.float64) + p["b2"]) == 0.0


def test_closed_form_single_token_user():
    batch, cfg, p = _tiny([1, 4], n_norm=5)
    out = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, None, p, cfg)
    hd = cfg.head_dim
    for h in range(cfg.num_heads):
        sl = slice(h * hd, (h + 1) * hd)
        s = float(out["Q"][0, sl] @ out["K"][0, sl]) + p["rab_pos"][0] + p["rab_time"][0]
        expect = s / (1.0 + math.exp(-s)) * out["V"][0, sl] / 5.0
        assert max_abs(out["O"][0, sl], expect) < 1e-15


def test_closed_form_zero_scores_give_beta_gate():
    """Q = K = 0 and rab = 0  =>  s = 0, SiLU(0) = 0, O = 0, Norm(O) = beta."""
    batch, cfg, p = _tiny([5, 7, 2])
    d = cfg.d_model
    p["w1"][2 * d:] = 0.0
    p["b1"][2 * d:] = 0.0
    p["rab_pos"][:] = 0.0
    p["rab_time"][:] = 0.0
    out = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, None, p, cfg)
    assert np.all(out["O"] == 0.0)
    X = batch.x.astype(np.float64)
    U = oracle.silu(X @ p["w1"][:d].T + p["b1"][:d])
    Y = (p["ln_beta"] * U) @ p["w2"].T + p["b2"] + X
    assert max_abs(out["Y"], Y) < 1e-13


@pytest.mark.parametrize("mask,ncand", [("causal", None), ("mfalcon", [3, 0, 5])])
def test_closed_form_constant_scores_give_masked_prefix_sums(mask, ncand):
    """Q = K = 0 and constant rab c  =>  O_i = SiLU(c)/n_norm * sum of visible V_j.

    causal: the running sum of V inside the user (a cumulative sum);
    M-FALCON candidate: the whole history plus its own V; history rows causal.
    """
    batch, cfg, p = _tiny([8, 4, 9], ncand=ncand, mask=mask, n_norm=10)
    d = cfg.d_model
    p["w1"][2 * d:] = 0.0
    p["b1"][2 * d:] = 0.0
    p["rab_pos"][:] = 0.375
    p["rab_time"][:] = 0.25
    out = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                            p, cfg)
    c = 0.625
    w = c / (1.0 + math.exp(-c)) / 10.0
    offs = batch.seq_offsets
    for b in range(3):
        lo, hi = int(offs[b]), int(offs[b + 1])
        Vb = out["V"][lo:hi]
        cs = np.cumsum(Vb, axis=0)
        nc = 0 if ncand is None else ncand[b]
        nh = (hi - lo) - nc
        for i in range(hi - lo):
            if i < nh:
                expect = w * cs[i]
            else:
                expect = w * (cs[nh - 1] if nh > 0 else 0.0) + w * Vb[i]
            assert max_abs(out["O"][lo + i], expect) < 1e-14


@pytest.mark.parametrize("mask,ncand", [("causal", None), ("mfalcon", [2, 4])])
def test_identity_phi_reduces_to_masked_matmul(mask, ncand):
    """With phi2 = identity, equation (2) is ((Q K^T + R) * M) V / n_norm.

    Checked with one dense torch matmul per padded user block, where R and the
    mask M are rebuilt here from their definitions.
    """
    batch, cfg, p = _tiny([6, 9], ncand=ncand, mask=mask, n_norm=7, d=8, H=1)
    X = batch.x.astype(np.float64)
    U, V, Q, K = oracle.f1_split(X, p["w1"], p["b1"], cfg.d_model)
    O = ho.pointwise_attention(Q, K, V, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                               p["rab_pos"], p["rab_time"], cfg, phi2=lambda s: s)
    offs = batch.seq_offsets
    for b in range(2):
        lo, hi = int(offs[b]), int(offs[b + 1])
        n = hi - lo
        nc = 0 if ncand is None else ncand[b]
        nh = n - nc
        R = np.zeros((n, n))
        M = np.zeros((n, n))
        for i in range(n):
            for j in range(n):
                cand = mask == "mfalcon" and i >= nh
                vis = (j < nh or j == i) if cand else (j <= i)
                rel = (0 if j == i else nh - j) if cand else i - j
                dt = max(int(batch.timestamps[lo + i]) - int(batch.timestamps[lo + j]), 0)
                tb = min(int(math.floor(math.log(1.0 + dt) / 0.301)), 127)
                R[i, j] = p["rab_pos"][min(max(rel, 0), 128)] + p["rab_time"][tb]
                M[i, j] = 1.0 if vis else 0.0
        S = torch.from_numpy(Q[lo:hi]) @ torch.from_numpy(K[lo:hi]).T + torch.from_numpy(R)
        ref = ((S * torch.from_numpy(M)) @ torch.from_numpy(V[lo:hi])) / 7.0
        assert max_abs(O[lo:hi], ref.numpy()) < 1e-12


# ---------------------------------------------------------------- bucket rules

def _exact_time_bucket(dt: int, div: float, nb: int) -> int:
    """floor(ln(1 + dt) / div) with 60 significant digits (div taken as its exact double)."""
    if dt <= 0:
        return 0
    ctx = decimal.Context(prec=60)
    q = ctx.divide(ctx.ln(decimal.Decimal(1 + dt)), decimal.Decimal(div))
    return min(int(q.to_integral_value(rounding=decimal.ROUND_FLOOR)), nb - 1)


def test_time_bucket_known_values():
    tb = lambda dt: int(oracle.time_bucket(np.array([dt]), 0.301, 128)[0])
    assert tb(0) == 0
    assert tb(-5) == 0                   # negative gaps clamp to 0
    assert tb(1) == 2                    # ln 2 / 0.301 = 2.30
    assert tb(2) == 3                    # ln 3 / 0.301 = 3.65
    assert tb(3600) == 27                # ln 3601 / 0.301 = 27.21
    assert tb(2 ** 62) == 127            # far past the last boundary: clamped
    assert tb(86400) == 37               # one day: ln 86401 / 0.301 = 37.77


def test_time_bucket_boundaries_match_exact_math():
    """At every bucket boundary exp(k * div) - 1 the fp64 rule agrees with 60-digit math.

    Exact agreement is required for gaps below 2^40 s (35,000 years), where
    neighbouring integer gaps differ in ln(1 + dt) / div by more than the fp64
    rounding of that quotient.  Above it the fp64 evaluation is the rule: it
    stays monotone and within one bucket of the exact value.
    """
    div = 0.301
    ctx = decimal.Context(prec=60)
    dts = []
    for k in range(1, 128):
        edge = ctx.subtract(ctx.exp(ctx.multiply(decimal.Decimal(k), decimal.Decimal(div))), 1)
        e = int(edge.to_integral_value(rounding=decimal.ROUND_FLOOR))
        dts += [max(e - 1, 0), e, e + 1, e + 2]
    dts = np.array(sorted(set(d for d in dts if d < 2 ** 62)), dtype=np.int64)
    got = oracle.time_bucket(dts, div, 128)
    want = np.array([_exact_time_bucket(int(d), div, 128) for d in dts])
    small = dts < 2 ** 40
    assert np.array_equal(got[small], want[small])
    assert np.all(np.abs(got - want) <= 1)
    assert np.all(np.diff(got) >= 0)
    # every bucket is reached except bucket 1 (ln 2 / 0.301 > 2: no integer gap)
    assert set(got[small].tolist()) == set(range(0, int(got[small].max()) + 1)) - {1}
    assert int(got[small].max()) >= 90 and int(got.max()) == 127


def test_position_bucket_clamps():
    rel = np.array([-3, 0, 1, 127, 128, 129, 10_000])
    assert oracle.position_bucket(rel, 128).tolist() == [0, 0, 1, 127, 128, 128, 128]
    assert oracle.position_bucket(rel, 1024).tolist() == [0, 0, 1, 127, 128, 129, 1024]


# ---------------------------------------------------------------- invariants

def test_causal_prefix_invariant():
    batch, cfg, p = _tiny([12, 9, 15], n_norm=16)
    full = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, None, p, cfg)["Y"]
    pref = 5
    offs = batch.seq_offsets
    keep = np.concatenate([np.arange(offs[b], offs[b] + pref) for b in range(3)])
    offs_p = np.arange(0, 3 * pref + 1, pref, dtype=np.int32)
    part = oracle.hstu_layer(batch.x[keep], offs_p, batch.timestamps[keep], None, p, cfg)["Y"]
    assert max_abs(part, full[keep]) < 1e-13


def test_per_user_results_independent_of_packing():
    batch, cfg, p = _tiny([7, 0, 11, 4], n_norm=12)
    full = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, None, p, cfg)["Y"]
    offs = batch.seq_offsets
    order = [2, 1, 3, 1, 0]        # permuted, with extra zero-length users
    rows, lens = [], []
    for b in order:
        rows.append(np.arange(offs[b], offs[b + 1]))
        lens.append(int(offs[b + 1] - offs[b]))
    rows = np.concatenate(rows)
    offs2 = wl.offsets_from_lengths(np.array(lens))
    y2 = oracle.hstu_layer(batch.x[rows], offs2, batch.timestamps[rows], None, p, cfg)["Y"]
    assert max_abs(y2, full[rows]) < 1e-13
    assert y2.shape[0] == full.shape[0]      # zero-length users add no rows


def test_mfalcon_candidates_do_not_see_each_other():
    nh, nc = 6, 5
    batch, cfg, p = _tiny([nh + nc, 4], ncand=[nc, 0], mask="mfalcon", n_norm=8)
    full = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                             p, cfg)["Y"]
    # drop candidates 1 and 3, permute the rest: remaining candidates unchanged
    keep_c = [4, 0, 2]
    rows = np.concatenate([np.arange(nh), nh + np.array(keep_c), np.arange(nh + nc, nh + nc + 4)])
    offs2 = np.array([0, nh + len(keep_c), nh + len(keep_c) + 4], dtype=np.int32)
    y2 = oracle.hstu_layer(batch.x[rows], offs2, batch.timestamps[rows],
                           np.array([len(keep_c), 0], np.int32), p, cfg)["Y"]
    assert max_abs(y2, full[rows]) < 1e-13
    # micro-batches of one candidate each give the same candidate rows
    for c in range(nc):
        rows = np.concatenate([np.arange(nh), [nh + c]])
        y1 = oracle.hstu_layer(batch.x[rows], np.array([0, nh + 1], np.int32),
                               batch.timestamps[rows], np.array([1], np.int32), p, cfg)["Y"]
        assert max_abs(y1[nh], full[nh + c]) < 1e-13


def test_mfalcon_history_equals_causal_and_zero_candidates_equal_causal():
    nh, nc = 7, 4
    batch, cfg, p = _tiny([nh + nc], ncand=[nc], mask="mfalcon", n_norm=9)
    full = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                             p, cfg)["Y"]
    cfg_c = oracle_cfg(cfg.d_model, cfg.num_heads, n_norm=9, mask="causal")
    hist = oracle.hstu_layer(batch.x[:nh], np.array([0, nh], np.int32), batch.timestamps[:nh],
                             None, p, cfg_c)["Y"]
    assert max_abs(full[:nh], hist) < 1e-13
    zero = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps,
                             np.array([0], np.int32), p, cfg)["Y"]
    caus = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, None, p, cfg_c)["Y"]
    assert max_abs(zero, caus) == 0.0


def test_no_softmax_row_sums_not_one():
    batch, cfg, p = _tiny([10], n_norm=1)
    rec = {}
    X = batch.x.astype(np.float64)
    U, V, Q, K = oracle.f1_split(X, p["w1"], p["b1"], cfg.d_model)
    ho.pointwise_attention(Q, K, V, batch.seq_offsets, batch.timestamps, None, p["rab_pos"],
                           p["rab_time"], cfg, record=rec)
    a = rec[0][0]
    sums = a.sum(axis=1)
    assert not np.allclose(sums, 1.0)
    # the weights are pointwise SiLU of the score: rescaling V by 2 doubles O
    O1 = ho.pointwise_attention(Q, K, V, batch.seq_offsets, batch.timestamps, None,
                                p["rab_pos"], p["rab_time"], cfg)
    O2 = ho.pointwise_attention(Q, K, 2 * V, batch.seq_offsets, batch.timestamps, None,
                                p["rab_pos"], p["rab_time"], cfg)
    assert max_abs(O2, 2 * O1) < 1e-14


def test_row_subset_equals_full_rows():
    batch, cfg, p = _tiny([9, 13], ncand=[3, 5], mask="mfalcon", n_norm=11)
    full = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                             p, cfg)
    rows = np.array([0, 4, 8, 9, 15, 21])
    part = oracle.hstu_layer(batch.x, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                             p, cfg, rows=rows)
    for key in ("O", "N", "G", "Y"):
        assert max_abs(part[key][rows], full[key][rows]) < 1e-14


def test_stack_is_layer_composition():
    batch = wl.make_custom_batch([5, 8], 8, 2, seed=11, num_layers=3, weight_scale=0.3)
    cfg = oracle_cfg(8, 2, n_norm=8)
    Y = batch.x.astype(np.float64)
    for lp in batch.layers:
        Y = oracle.hstu_layer(Y, batch.seq_offsets, batch.timestamps, None, params_dict(lp), cfg)["Y"]
    S = oracle.hstu_stack(batch.x, batch.seq_offsets, batch.timestamps, None,
                          [params_dict(lp) for lp in batch.layers], cfg)
    assert max_abs(S, Y) == 0.0


def test_visible_pairs_counts():
    offs = np.array([0, 4, 4, 10], np.int32)
    assert oracle.visible_pairs(offs, None, "causal") == 10 + 21
    # user of 10: 6 history (21 pairs) + 4 candidates each seeing 6 + self
    assert oracle.visible_pairs(np.array([0, 10]), np.array([4]), "mfalcon") == 21 + 4 * 7


# ---------------------------------------------------------------- planted mistakes

def _mutant_results(monkeypatch, name, fn):
    monkeypatch.setattr(ho, name, fn)
    batch = wl.make_custom_batch([6, 9], 8, 2, seed=5, num_candidates=[0, 3], pos_buckets=9,
                                 time_buckets=20, weight_scale=0.7, rab_scale=1.5,
                                 random_affine=True, timestamp_gap=5.0)
    cfg = oracle_cfg(8, 2, pos_clamp=8, time_buckets=20, n_norm=0, mask="mfalcon")
    return _run_both(batch, cfg)


@pytest.mark.parametrize("name,mutant", [
    # split order swapped (Q and K exchanged)
    ("f1_split", lambda X, W1, b1, d: (lambda Z: (Z[:, :d], Z[:, d:2 * d], Z[:, 3 * d:], Z[:, 2 * d:3 * d]))(
        ho.silu(X @ W1.T + b1))),
    # time bias dropped
    ("user_rab", lambda ts, q, rel, rp, rt, cfg: (rp[ho.position_bucket(rel, cfg.pos_clamp)],
                                                  None, None)),
    # off-by-one time bucket
    ("time_bucket", lambda dt, div, nb: np.minimum(np.floor(np.log(2.0 + np.maximum(dt, 0)) / div),
                                                   nb - 1).astype(np.int64)),
    # causal mask including the next token
    ("user_visibility", lambda n, nc, mask, q=None: (lambda i, j: ((j <= i + 1), (i - j)))(
        np.arange(n)[:, None], np.arange(n)[None, :])),
    # LayerNorm with unbiased variance
    ("layer_norm", lambda O, g, b, eps: (O - O.mean(1, keepdims=True)) /
        np.sqrt(O.var(1, ddof=1, keepdims=True) + eps) * g + b),
])
def test_planted_mistakes_are_caught(monkeypatch, name, mutant):
    o, b = _mutant_results(monkeypatch, name, mutant)
    worst = max(max_abs(o[k], b[k]) for k in ("U", "V", "Q", "K", "O", "Y"))
    assert worst > 1e-6, f"mutant {name} was not detected"
