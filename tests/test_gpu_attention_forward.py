"""GPU: hstu_attention_forward, the attention step alone on the handle.

Given the U|V|Q|K that hstu_layer_forward produced, the entry point must
return that call's attention output O (equation (2), already divided by
n_norm) bit for bit -- the same schedule and kernel -- and O must match the
oracle's equation (2) evaluated on the same U|V|Q|K within the per-element
bound of the forward parity tests."""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_params, teacher_forced_attention
from helpers import oracle_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("compute,mask,lengths,ncand,d,H", [
    ("bf16", "causal", [1, 127, 129, 300, 0, 257], None, 256, 2),
    ("bf16", "mfalcon", [300, 140, 260], [100, 140, 129], 256, 4),
    ("fp32", "causal", [20, 104, 100, 53], None, 64, 2),
])
def test_attention_forward_equals_the_layer_step(compute, mask, lengths, ncand, d, H):
    batch = wl.make_custom_batch(lengths, d, H, seed=5 + sum(lengths), num_candidates=ncand,
                                 weight_scale=0.05, rab_scale=0.5)
    n_norm = 0 if mask == "causal" else 512
    dt = hstu.HSTU_DTYPE_BF16 if compute == "bf16" else hstu.HSTU_DTYPE_FP32
    cfg = hstu.make_config(d, H, io_dtype=dt, compute_dtype=dt, n_norm=n_norm, pos_buckets=129,
                           pos_clamp=128, time_buckets=128, time_log_div=0.301, ln_eps=1e-5,
                           max_tokens=batch.total_tokens, max_users=batch.num_users)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, compute, compute, "cuda:0")
    T = batch.total_tokens
    mode = hstu.HSTU_MASK_MFALCON if mask == "mfalcon" else hstu.HSTU_MASK_CAUSAL
    out = torch.empty_like(db.x)
    h.forward(db, out, mode)
    uvqk = h.intermediate(hstu.HSTU_TENSOR_UVQK, T).clone()
    av_ref = h.intermediate(hstu.HSTU_TENSOR_AV, T).clone()
    av = torch.full_like(av_ref, float("nan"))
    lp = db.layers[0]
    hstu.hstu_attention_forward(h.h, uvqk, T, db.seq_offsets, db.num_users, db.timestamps, mode,
                                db.num_candidates, lp.rab_pos, lp.rab_time, av,
                                torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.device_error() == 0
    h.close()
    assert torch.equal(av, av_ref)
    # against the oracle's equation (2) on the same U|V|Q|K
    U = uvqk.double().cpu().numpy()
    ocfg = oracle_cfg(d, H, n_norm=n_norm, mask=mask)
    ref, ref_abs = teacher_forced_attention(U, batch, ocfg, oracle_params(batch.layers[0], compute),
                                            with_abs=True)
    got = av.double().cpu().numpy()
    if compute == "bf16":
        rms = float(np.sqrt(np.mean(ref * ref)))
        assert np.all(np.abs(got - ref) <= 2.0 ** -7 * ref_abs + 1e-6 * rms)
    else:
        assert np.max(np.abs(got - ref)) <= 1e-4


def test_attention_forward_of_an_empty_batch_launches_nothing():
    cfg = hstu.make_config(256, 2, io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16,
                           n_norm=256, pos_buckets=129, pos_clamp=128, time_buckets=128,
                           time_log_div=0.301, ln_eps=1e-5, max_tokens=16, max_users=2)
    h = runtime.Handle(cfg, 0)
    offs = torch.zeros(3, dtype=torch.int32, device="cuda:0")
    hstu.hstu_attention_forward(h.h, None, 0, offs, 2, None, hstu.HSTU_MASK_CAUSAL, None, None,
                                None, None, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.device_error() == 0
    h.close()
