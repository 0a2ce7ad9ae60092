"""GPU: backward of one HSTU layer against the fp64 oracle.

The forward runs on the GPU (its U|V|Q|K and O are the inputs the backward
reads), the backward gets a random dY, and every gradient is compared with
the oracle's hstu_layer_backward of the same X and dY.  Each side carries
its own forward: the GPU's bf16 roundings of X, U|V|Q|K, P, G and of the
backward's products (dY, dO, dS, dH1 and the transposed operands, 2^-9
relative each) all reach the gradients.  Re-running these three cases in
fp64 with every one of those roundings applied (and the hardware sigmoid's
error drawn uniformly within its bound) gives at most 4.6% of RMS (the
time-bias gradient, fp32 stream; the weight gradients reach 3.4%), so the
bound is per tensor: max-abs <= 1e-1 x RMS(reference)."""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_params
from helpers import oracle_cfg

pytestmark = pytest.mark.gpu

KEYS = ("w1", "b1", "w2", "b2", "ln_gamma", "ln_beta", "rab_pos", "rab_time")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rel(g, r):
    r = np.asarray(r, np.float64)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    return float(np.max(np.abs(np.asarray(g, np.float64) - r))) / max(rms, 1e-30)


@pytest.mark.parametrize("storage,mask,lengths,ncand,H", [
    ("bf16", "causal", [1, 127, 129, 300, 0, 5], None, 2),
    ("fp32", "causal", [255, 257], None, 4),
    ("bf16", "mfalcon", [300, 140, 260], [100, 140, 129], 4),
])
def test_layer_backward_matches_the_oracle(storage, mask, lengths, ncand, H):
    d = 256
    batch = wl.make_custom_batch(lengths, d, H, seed=3 * sum(lengths) + H, num_candidates=ncand,
                                 weight_scale=0.05, rab_scale=1.0, random_affine=True,
                                 timestamp_gap=900.0)
    n_norm = 512
    cfg = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16 if storage == "bf16" else hstu.HSTU_DTYPE_FP32,
                           compute_dtype=hstu.HSTU_DTYPE_BF16, n_norm=n_norm, pos_buckets=129,
                           pos_clamp=128, time_buckets=128, time_log_div=0.301, ln_eps=1e-5,
                           max_tokens=batch.total_tokens, max_users=len(lengths))
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, storage, "bf16", "cuda:0")
    T = batch.total_tokens
    mode = hstu.HSTU_MASK_MFALCON if mask == "mfalcon" else hstu.HSTU_MASK_CAUSAL
    y = torch.empty_like(db.x)
    h.forward(db, y, mode)
    uvqk = h.intermediate(hstu.HSTU_TENSOR_UVQK, T)
    av = h.intermediate(hstu.HSTU_TENSOR_AV, T)
    rng = np.random.default_rng(11)
    dY_np = rng.normal(size=(T, d)).astype(np.float32)
    dY = torch.from_numpy(dY_np).to("cuda:0", db.x.dtype)
    dX = torch.empty_like(dY)
    f32 = dict(dtype=torch.float32, device="cuda:0")
    grads = {"w1": torch.empty((4 * d, d), **f32), "b1": torch.empty(4 * d, **f32),
             "w2": torch.empty((d, d), **f32), "b2": torch.empty(d, **f32),
             "ln_gamma": torch.empty(d, **f32), "ln_beta": torch.empty(d, **f32),
             "rab_pos": torch.empty(129, **f32), "rab_time": torch.empty(128, **f32)}
    hstu.hstu_layer_backward(h.h, db.x, uvqk, av, dY, T, db.seq_offsets, db.num_users,
                             db.timestamps, db.layers[0].struct(), mode, db.num_candidates, dX,
                             grads, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.device_error() == 0
    h.close()
    X = wl.round_to_storage(batch.x, storage).astype(np.float64)
    dYr = dY.double().cpu().numpy()
    ref = oracle.hstu_layer_backward(X, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                                     oracle_params(batch.layers[0], "bf16"),
                                     oracle_cfg(d, H, n_norm=n_norm, mask=mask), dYr)
    assert _rel(dX.double().cpu().numpy(), ref["X"]) <= 1e-1
    for k in KEYS:
        assert _rel(grads[k].double().cpu().numpy(), ref[k]) <= 1e-1, k
