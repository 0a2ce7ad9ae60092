"""GPU: the attention backward at the benchmark's full size (8 users x 8192
tokens, d 1024 = 8 heads x 128, the 24-layer stack's layer 0), in the launch
configuration `bench.py --attn-bwd` times, checked on sampled outputs.

* dQ, dK and dV of user 0 (all 8,192 rows) on heads 0 and 7 against the
  oracle's pointwise_attention_backward run on that user alone: a user's
  gradients depend on its own rows only, and each head's on its own columns
  (plus the shared bias tables), so the oracle sees a one-user, two-head
  problem.  The per-element bounds are those of the small teacher-forced
  cases (test_gpu_attention_backward), evaluated on the same sample.
* The bias-table gradients of the whole batch through an identity that holds
  at any size: every visible (query, key, head) adds its dS to exactly one
  position entry and one time entry, so both tables sum to the same total.
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from helpers import cfg_for_workload
from test_gpu_attention_backward import _bounds, _rms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


class _OneUser:
    """The seq_offsets / timestamps / num_candidates view of user 0 alone."""

    def __init__(self, batch, n):
        self.seq_offsets = np.array([0, n], dtype=np.int64)
        self.timestamps = np.asarray(batch.timestamps[:n])
        self.num_candidates = np.zeros(1, dtype=np.int32)


def test_attention_backward_full_size_sampled():
    w = wl.WORKLOADS[3]
    batch = wl.make_batch(w, num_layers=1)
    T, d, H, hd = batch.total_tokens, w.d_model, w.num_heads, w.head_dim
    cfg = runtime.config_for(w, T, batch.num_users)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, w.storage, w.compute, "cuda:0")
    mode = runtime.mask_mode_of(w)
    y = torch.empty_like(db.x)
    h.forward(db, y, mode)
    uvqk = h.intermediate(hstu.HSTU_TENSOR_UVQK, T)
    dev = torch.device("cuda", 0)
    dO = torch.randn((T, d), generator=torch.Generator(device=dev).manual_seed(3), device=dev,
                     dtype=torch.float32).to(torch.bfloat16)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty((T, d), **f32) for _ in range(3))
    g_pos = torch.empty(w.pos_buckets, **f32)
    g_time = torch.empty(w.time_buckets, **f32)
    lp = db.layers[0]
    hstu.hstu_attention_backward(h.h, uvqk, dO, T, db.seq_offsets, db.num_users, db.timestamps,
                                 mode, db.num_candidates, lp.rab_pos, lp.rab_time, dq, dk, dv,
                                 g_pos, g_time, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.device_error() == 0
    h.close()

    # the bias tables: both sum every visible pair's dS once
    gp = g_pos.double().cpu().numpy()
    gt = g_time.double().cpu().numpy()
    scale = np.abs(gp).sum() + np.abs(gt).sum()
    assert scale > 0.0
    assert abs(gp.sum() - gt.sum()) <= 1e-4 * scale

    # user 0, heads 0 and 7, against the oracle
    n = int(batch.seq_offsets[1] - batch.seq_offsets[0])
    assert n == 8192
    heads = [0, H - 1]
    cols = np.concatenate([np.arange(k * hd, (k + 1) * hd) for k in heads])
    U = uvqk[:n].double().cpu().numpy()
    V, Q, K = (U[:, off + cols] for off in (d, 2 * d, 3 * d))
    dOn = dO[:n].double().cpu().numpy()[:, cols]
    ocfg = cfg_for_workload(w)
    ocfg = type(ocfg)(**{**ocfg.__dict__, "d_model": len(cols), "num_heads": len(heads)})
    one = _OneUser(batch, n)
    rp = batch.layers[0].rab_pos.astype(np.float64)
    rt = batch.layers[0].rab_time.astype(np.float64)
    rdq, rdk, rdv, _, _ = oracle.pointwise_attention_backward(
        Q, K, V, dOn, one.seq_offsets, one.timestamps, one.num_candidates, rp, rt, ocfg)
    bq, bk, bv, _, _ = _bounds(Q, K, V, dOn, one, ocfg, rp, rt)
    got = {"dq": dq, "dk": dk, "dv": dv}
    for name, ref, bound in (("dq", rdq, bq), ("dk", rdk, bk), ("dv", rdv, bv)):
        g = got[name][:n].double().cpu().numpy()[:, cols]
        err = np.abs(g - ref)
        assert np.all(err <= bound + 1e-6 * _rms(ref)), (name, float(err.max()), float(_rms(ref)))
