"""GPU: backward of the attention step against the oracle, teacher-forced.

The kernel gets the forward's own U|V|Q|K (bf16, from a forward on the same
handle) and a bf16 dO; the oracle's pointwise_attention_backward evaluates
the exact gradients on those same values in fp64.  Per-element bounds from
the kernel's arithmetic:
  dV = sum_i a_ij dO_i with a rounded to bf16 (2^-9) and sigmoid through the
       hardware tanh (absolute error below 2^-11):
       |err| <= 2^-7 sum_i |a_ij| |dO_i| + 1e-6 RMS
  dS = vis dA SiLU'(s) / n_norm, SiLU' = sig (1 + s (1 - sig)): a sigmoid
       error e moves SiLU' by at most e (1 + 2|s|); dS is then rounded to
       bf16 for the products, so per pair
       |err dS| <= 2^-8 |dS| + 2^-11 (1 + 2|s|) |dA| / n_norm  (=: eps_ij)
  dQ_i = sum_j dS_ij k_j:  |err| <= sum_j eps_ij |k_j| + 2^-9 sum_j |dS_ij k_j| + 1e-6 RMS
  dK_j = sum_i dS_ij q_i:  the same with q
  bias tables (fp32 sums of the unrounded dS): |err| <= sum of (eps_ij - 2^-8 |dS_ij|)
       over the pairs reading the entry, + 1e-5 RMS
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import hstu_backward as hb
from oracle import hstu_oracle as ho
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from helpers import oracle_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _bounds(Q, K, V, dO, batch, cfg, rab_pos, rab_time):
    """Per-element error bounds of dQ, dK, dV and of the bias tables."""
    T, d = Q.shape
    H, hd = cfg.num_heads, cfg.head_dim
    offs = batch.seq_offsets.astype(np.int64)
    nn = ho.effective_n_norm(cfg, offs[1:] - offs[:-1])
    bq, bk, bv = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    bpos, btime = np.zeros_like(rab_pos), np.zeros_like(rab_time)
    for b in range(len(offs) - 1):
        lo, hi = int(offs[b]), int(offs[b + 1])
        n = hi - lo
        if n == 0:
            continue
        n_c = int(batch.num_candidates[b]) if cfg.mask == "mfalcon" else 0
        vis, rel = ho.user_visibility(n, n_c, cfg.mask)
        rab, pidx, tidx = ho.user_rab(batch.timestamps[lo:hi], np.arange(n), rel, rab_pos,
                                      rab_time, cfg)
        for h in range(H):
            c = slice(h * hd, (h + 1) * hd)
            s = Q[lo:hi, c] @ K[lo:hi, c].T + rab
            a = np.where(vis, ho.silu(s) / nn, 0.0)
            da = dO[lo:hi, c] @ V[lo:hi, c].T
            ds = np.where(vis, da * hb.silu_grad(s) / nn, 0.0)
            e_s = np.where(vis, 2.0 ** -11 * (1 + 2 * np.abs(s)) * np.abs(da) / nn, 0.0)
            eps = 2.0 ** -8 * np.abs(ds) + e_s
            bv[lo:hi, c] += 2.0 ** -7 * (np.abs(a).T @ np.abs(dO[lo:hi, c]))
            bq[lo:hi, c] += eps @ np.abs(K[lo:hi, c]) + 2.0 ** -9 * (np.abs(ds) @ np.abs(K[lo:hi, c]))
            bk[lo:hi, c] += eps.T @ np.abs(Q[lo:hi, c]) + 2.0 ** -9 * (np.abs(ds).T @ np.abs(Q[lo:hi, c]))
            np.add.at(bpos, pidx[vis], e_s[vis])
            np.add.at(btime, tidx[vis], e_s[vis])
    return bq, bk, bv, bpos, btime


def _rms(x):
    return float(np.sqrt(np.mean(np.asarray(x, np.float64) ** 2))) if np.size(x) else 0.0


@pytest.mark.parametrize("mask,lengths,ncand,H,n_norm", [
    ("causal", [1, 127, 128, 129, 300, 0, 5], None, 2, 512),
    ("causal", [255, 256, 257], None, 4, 512),
    ("mfalcon", [300, 140, 260], [100, 140, 129], 4, 512),
    # n_norm = the longest user of the batch, found on the device by the schedule
    ("causal", [40, 300, 0, 129], None, 2, 0),
    # a long user: most half tiles take the constant-bias path (every pair visible,
    # clamped position, one time bucket per row)
    ("causal", [1100, 37], None, 2, 1200),
])
def test_attention_backward_teacher_forced(mask, lengths, ncand, H, n_norm):
    d = 256
    batch = wl.make_custom_batch(lengths, d, H, seed=sum(lengths) + H, num_candidates=ncand,
                                 weight_scale=0.05, rab_scale=1.0, random_affine=True,
                                 timestamp_gap=900.0)
    cfg_gpu = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16,
                               compute_dtype=hstu.HSTU_DTYPE_BF16, n_norm=n_norm, pos_buckets=129,
                               pos_clamp=128, time_buckets=128, time_log_div=0.301, ln_eps=1e-5,
                               max_tokens=batch.total_tokens, max_users=len(lengths))
    h = runtime.Handle(cfg_gpu, 0)
    db = runtime.to_device(batch, "bf16", "bf16", "cuda:0")
    out = torch.empty_like(db.x)
    mode = hstu.HSTU_MASK_MFALCON if mask == "mfalcon" else hstu.HSTU_MASK_CAUSAL
    h.forward(db, out, mode)
    T = batch.total_tokens
    uvqk = h.intermediate(hstu.HSTU_TENSOR_UVQK, T)
    rng = np.random.default_rng(7)
    dO = torch.from_numpy(rng.normal(size=(T, d)).astype(np.float32)).to("cuda:0", torch.bfloat16)
    dq = torch.empty((T, d), dtype=torch.float32, device="cuda:0")
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    lp = db.layers[0]
    g_pos = torch.empty(129, dtype=torch.float32, device="cuda:0")
    g_time = torch.empty(128, dtype=torch.float32, device="cuda:0")
    hstu.hstu_attention_backward(h.h, uvqk, dO, T, db.seq_offsets, db.num_users, db.timestamps,
                                 mode, db.num_candidates, lp.rab_pos, lp.rab_time, dq, dk, dv,
                                 g_pos, g_time, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.device_error() == 0
    h.close()
    U = uvqk.double().cpu().numpy()
    V, Q, K = U[:, d:2 * d], U[:, 2 * d:3 * d], U[:, 3 * d:]
    dOn = dO.double().cpu().numpy()
    cfg = oracle_cfg(d, H, n_norm=n_norm, mask=mask)
    rp = batch.layers[0].rab_pos.astype(np.float64)
    rt = batch.layers[0].rab_time.astype(np.float64)
    rdq, rdk, rdv, rpos, rtime = oracle.pointwise_attention_backward(
        Q, K, V, dOn, batch.seq_offsets, batch.timestamps, batch.num_candidates, rp, rt, cfg)
    bq, bk, bv, bpos, btime = _bounds(Q, K, V, dOn, batch, cfg, rp, rt)
    got = {"dq": dq, "dk": dk, "dv": dv}
    for name, ref, bound in (("dq", rdq, bq), ("dk", rdk, bk), ("dv", rdv, bv)):
        g = got[name].double().cpu().numpy()
        assert np.all(np.abs(g - ref) <= bound + 1e-6 * _rms(ref)), name
    gp = g_pos.double().cpu().numpy()
    gt = g_time.double().cpu().numpy()
    assert np.all(np.abs(gp - rpos) <= bpos + 1e-5 * _rms(rpos) + 1e-7)
    assert np.all(np.abs(gt - rtime) <= btime + 1e-5 * _rms(rtime) + 1e-7)
