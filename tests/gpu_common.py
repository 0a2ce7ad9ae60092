"""Helpers of the GPU parity tests: run the C-ABI path and the oracle on the
same seeded inputs (the oracle sees exactly the values stored in HBM)."""
import numpy as np
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from helpers import cfg_for_workload, oracle_cfg


def oracle_params(lp, compute):
    """Layer parameters exactly as the GPU holds them, promoted to float64."""
    p = {}
    for k in ("w1", "w2"):
        p[k] = wl.round_to_storage(getattr(lp, k), compute).astype(np.float64)
    for k in ("b1", "b2", "rab_pos", "rab_time", "ln_gamma", "ln_beta"):
        p[k] = np.asarray(getattr(lp, k), dtype=np.float32).astype(np.float64)
    return p


def gpu_run(batch, storage, compute, *, d, H, n_norm, mask, pos_buckets=129, pos_clamp=128,
            time_buckets=128, div=0.301, eps=1e-5, layers=None, want=("UVQK", "AV", "G")):
    """Runs the layer stack on cuda:0 and returns numpy float64 results."""
    cfg = hstu.make_config(
        d, H, io_dtype=hstu.HSTU_DTYPE_BF16 if storage == "bf16" else hstu.HSTU_DTYPE_FP32,
        compute_dtype=hstu.HSTU_DTYPE_BF16 if compute == "bf16" else hstu.HSTU_DTYPE_FP32,
        n_norm=n_norm, pos_buckets=pos_buckets, pos_clamp=pos_clamp, time_buckets=time_buckets,
        time_log_div=div, ln_eps=eps, max_tokens=max(batch.total_tokens, 1),
        max_users=max(batch.num_users, 1))
    handle = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, storage, compute, "cuda:0")
    T = batch.total_tokens
    out = torch.empty_like(db.x)
    mode = hstu.HSTU_MASK_MFALCON if mask == "mfalcon" else hstu.HSTU_MASK_CAUSAL
    handle.forward(db, out, mode, layers=layers)
    res = {"Y": out.double().cpu().numpy()}
    for name in want:
        which = {"UVQK": hstu.HSTU_TENSOR_UVQK, "AV": hstu.HSTU_TENSOR_AV,
                 "G": hstu.HSTU_TENSOR_G}[name]
        if T > 0:
            res[name] = handle.intermediate(which, T).double().cpu().numpy()
    torch.cuda.synchronize()
    res["error"] = handle.device_error()
    handle.close()
    return res


def oracle_inputs(batch, storage):
    return wl.round_to_storage(batch.x, storage).astype(np.float64)


def teacher_forced_attention(uvqk_gpu, batch, cfg, params, with_abs=False):
    """The oracle's equation (2) evaluated on the GPU's own U,V,Q,K.

    With ``with_abs`` also returns sum_j |a_ij| |v_j| (the scale of the
    rounding error of each output element)."""
    d = cfg.d_model
    V = uvqk_gpu[:, d:2 * d]
    Q = uvqk_gpu[:, 2 * d:3 * d]
    K = uvqk_gpu[:, 3 * d:]
    args = (batch.seq_offsets, batch.timestamps, batch.num_candidates, params["rab_pos"],
            params["rab_time"], cfg)
    O = oracle.pointwise_attention(Q, K, V, *args)
    if not with_abs:
        return O
    O_abs = oracle.pointwise_attention(Q, K, np.abs(V), *args,
                                       phi2=lambda s: np.abs(oracle.silu(s)))
    return O, O_abs


def rel_err(gpu, ref):
    """max |gpu - ref| / RMS(ref)."""
    ref = np.asarray(ref, np.float64)
    r = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - ref))) / max(r, 1e-30)
