"""GPU: backward of one HSTU layer at the benchmark's full size (8 users x 8192
tokens, d 1024 = 8 heads x 128, fp32 residual stream: layer 0 of the 24-layer
stack), checked on outputs the oracle can compute and on closed forms.

* dX of user 0's first 2048 rows.  dY is zero on the rest of user 0, so no
  gradient reaches those rows from later queries (n_norm is fixed and the
  LayerNorm is per row): their dX is the oracle's layer backward of the
  2048-token prefix alone.  Bound of the small cases: max-abs <= 1e-1 RMS.
* db2 = the column sums of dY and dW2 = dY^T G (G = LN(O) * U, the forward's
  own gate output), both over all 65,536 rows, against float64 sums and
  products.  The layer backward multiplies dY rounded to bf16 (to nearest),
  so the reference product takes dY rounded the same way; what is left is
  the fp32 accumulation of the products, well inside 1e-3 RMS.
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_params
from helpers import cfg_for_workload
from test_gpu_layer_backward import _rel

pytestmark = pytest.mark.gpu

PREFIX = 2048


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_layer_backward_full_size_sampled():
    w = wl.WORKLOADS[3]
    batch = wl.make_batch(w, num_layers=1)
    T, d = batch.total_tokens, w.d_model
    n0 = int(batch.seq_offsets[1] - batch.seq_offsets[0])
    assert n0 == 8192 and w.storage == "fp32"
    cfg = runtime.config_for(w, T, batch.num_users)
    h = runtime.Handle(cfg, 0)
    dev = torch.device("cuda", 0)
    db = runtime.to_device(batch, w.storage, w.compute, dev)
    mode = runtime.mask_mode_of(w)
    y = torch.empty_like(db.x)
    h.forward(db, y, mode)
    uvqk = h.intermediate(hstu.HSTU_TENSOR_UVQK, T)
    av = h.intermediate(hstu.HSTU_TENSOR_AV, T)
    G = h.intermediate(hstu.HSTU_TENSOR_G, T)
    dY = torch.randn((T, d), generator=torch.Generator(device=dev).manual_seed(5), device=dev,
                     dtype=torch.float32)
    dY[PREFIX:n0] = 0.0
    dX = torch.empty_like(dY)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"w1": torch.empty((4 * d, d), **f32), "b1": torch.empty(4 * d, **f32),
             "w2": torch.empty((d, d), **f32), "b2": torch.empty(d, **f32),
             "ln_gamma": torch.empty(d, **f32), "ln_beta": torch.empty(d, **f32),
             "rab_pos": torch.empty(w.pos_buckets, **f32),
             "rab_time": torch.empty(w.time_buckets, **f32)}
    hstu.hstu_layer_backward(h.h, db.x, uvqk, av, dY, T, db.seq_offsets, db.num_users,
                             db.timestamps, db.layers[0].struct(), mode, db.num_candidates, dX,
                             grads, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.device_error() == 0
    h.close()

    # closed forms over the whole batch
    dY64 = dY.double()
    assert _rel(grads["b2"].double().cpu().numpy(), dY64.sum(0).cpu().numpy()) <= 1e-3
    dW2 = (dY.to(torch.bfloat16).double().t() @ G.double()).cpu().numpy()
    assert _rel(grads["w2"].double().cpu().numpy(), dW2) <= 1e-3

    # dX of user 0's prefix against the oracle on that prefix alone
    X = wl.round_to_storage(batch.x[:PREFIX], w.storage).astype(np.float64)
    ref = oracle.hstu_layer_backward(X, np.array([0, PREFIX]), batch.timestamps[:PREFIX],
                                     np.zeros(1, dtype=np.int32),
                                     oracle_params(batch.layers[0], w.compute),
                                     cfg_for_workload(w), dY[:PREFIX].double().cpu().numpy())
    assert _rel(dX[:PREFIX].double().cpu().numpy(), ref["X"]) <= 1e-1
