"""Shared test helpers: oracle configs and parameter plumbing (no layer arithmetic)."""
import numpy as np

from oracle import OracleConfig


def oracle_cfg(d, H, *, pos_clamp=128, time_buckets=128, div=0.301, n_norm=0, eps=1e-5,
               mask="causal"):
    return OracleConfig(d_model=d, num_heads=H, head_dim=d // H, pos_clamp=pos_clamp,
                        time_buckets=time_buckets, time_log_div=div, n_norm=n_norm,
                        ln_eps=eps, mask=mask)


def cfg_for_workload(w):
    return OracleConfig(d_model=w.d_model, num_heads=w.num_heads, head_dim=w.head_dim,
                        pos_clamp=w.pos_clamp, time_buckets=w.time_buckets,
                        time_log_div=w.time_log_div, n_norm=w.n_norm, ln_eps=w.ln_eps,
                        mask=w.mask)


def params_dict(lp):
    return {k: np.asarray(getattr(lp, k), dtype=np.float64)
            for k in ("w1", "b1", "w2", "b2", "rab_pos", "rab_time", "ln_gamma", "ln_beta")}


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def rms(a):
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0
