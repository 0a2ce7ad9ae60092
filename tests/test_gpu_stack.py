"""GPU parity of the 24-layer stack at full size: 8 users x 8192 tokens,
d 1024, 8 heads x 128, fp32 residual stream, bf16 tensor-core operands.

* Per layer (the unit the layer tolerance is defined on): every layer's GPU
  output is compared with the oracle's layer applied to that layer's GPU input,
  on sampled rows of every one of the 8 full-length users (the oracle computes
  the rows one by one from the user's whole key range; the samples always hold
  rows 0, 1, 127, 128, 1023, 1024, 4095, 4096 and n-1, the edges of the 128-row
  tiles and of the 256-row tile pairs): max-abs <= 2e-2 x RMS per layer and user.
* The stack call that the benchmark times gives bit-identical output to the
  layer-by-layer calls checked above.
* Free-running: the last layer's output on the first 1024 tokens of all eight
  users against the oracle's own 24-layer run on those prefixes (exact by
  causality, n_norm held at 8192).  Per-layer bf16 rounding of the operands
  compounds through the residual stream, so this bound is 6e-2 x RMS:
  emulating the kernels' rounding points on the CPU gives 0.038 x RMS for this
  stack.

Both figures are printed (run with -s to see them).
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import build, hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_params, rel_err
from helpers import cfg_for_workload

pytestmark = pytest.mark.gpu

EDGE_ROWS = (0, 1, 127, 128, 1023, 1024, 4095, 4096)
RANDOM_ROWS = 8


def _sample_rows(n, seed):
    rng = np.random.default_rng(seed)
    fixed = [r for r in EDGE_ROWS if r < n] + [n - 1]
    return np.unique(np.concatenate([fixed, rng.integers(0, n, size=RANDOM_ROWS)]))


@pytest.fixture(scope="module")
def stack_run():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    w = wl.WORKLOADS[3]
    batch = wl.make_batch(w)
    cfg = runtime.config_for(w, batch.total_tokens, batch.num_users)
    ocfg = cfg_for_workload(w)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, w.storage, w.compute, "cuda:0")
    users = range(batch.num_users)
    rows = {u: _sample_rows(int(batch.seq_offsets[u + 1] - batch.seq_offsets[u]), 100 + u)
            for u in users}
    # per_layer[l][u] = max-abs / RMS of layer l's output on user u's sampled rows
    per_layer = np.zeros((w.num_layers, batch.num_users))
    cur = db.x.clone()
    for l in range(w.num_layers):
        nxt = torch.empty_like(cur)
        h.forward(db, nxt, hstu.HSTU_MASK_CAUSAL, layers=[db.layers[l]], x=cur)
        x_in = cur.double().cpu().numpy()
        y_gpu = nxt.double().cpu().numpy()
        p = oracle_params(batch.layers[l], w.compute)
        for u in users:
            lo, hi = int(batch.seq_offsets[u]), int(batch.seq_offsets[u + 1])
            n = hi - lo
            r = rows[u]
            ref = oracle.hstu_layer(x_in[lo:hi], np.array([0, n], dtype=np.int32),
                                    batch.timestamps[lo:hi], None, p, ocfg, rows=r)
            per_layer[l, u] = rel_err(y_gpu[lo:hi][r], ref["Y"][r])
        cur = nxt
    stacked = torch.empty_like(db.x)
    h.forward(db, stacked, hstu.HSTU_MASK_CAUSAL)
    torch.cuda.synchronize()
    err = h.device_error()
    result = dict(w=w, batch=batch, per_layer=per_layer, rows=rows,
                  same=bool(torch.equal(stacked, cur)), final=stacked.double().cpu().numpy(),
                  error=err)
    h.close()
    return result


def test_stack_call_equals_layer_sequence(stack_run):
    assert stack_run["error"] == 0
    assert stack_run["same"]


def test_every_layer_matches_the_oracle_on_every_user(stack_run):
    e = stack_run["per_layer"]
    n_rows = sum(len(r) for r in stack_run["rows"].values())
    l, u = np.unravel_index(int(np.argmax(e)), e.shape)
    print(f"per-layer max-abs/RMS over 24 layers x 8 users ({n_rows} rows per layer): "
          f"worst {e.max():.4f} (layer {l}, user {u}), median {np.median(e):.4f}")
    assert e.max() <= 2e-2, f"layer {l}, user {u}: max-abs / RMS = {e.max():.4f}"


def test_free_running_prefix_of_the_stack(stack_run):
    w, batch = stack_run["w"], stack_run["batch"]
    cfg = cfg_for_workload(w)
    prefix, users = 1024, list(range(batch.num_users))
    rows = np.concatenate([np.arange(batch.seq_offsets[u], batch.seq_offsets[u] + prefix)
                           for u in users])
    offs = np.arange(0, prefix * len(users) + 1, prefix, dtype=np.int32)
    params = [oracle_params(lp, w.compute) for lp in batch.layers]
    ref = oracle.hstu_stack(batch.x[rows].astype(np.float64), offs, batch.timestamps[rows], None,
                            params, cfg)
    e = rel_err(stack_run["final"][rows], ref)
    print(f"free-running 24-layer max-abs/RMS on 8 x 1024-token prefixes: {e:.4f}")
    assert e <= 6e-2
