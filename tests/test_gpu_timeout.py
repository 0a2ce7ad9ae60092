"""GPU: the bounded-wait failure path, exercised without a fault.

Every pipeline wait of the tensor-core kernels gives up after a bound of SM
cycles.  With the bound set to one cycle every f1 / attention / f2 launch of a
tiny layer gives up at its first wait that is not already satisfied: the
handle's error word must then carry HSTU_DEVERR_TIMEOUT (the kernels still
drain their own copies and MMAs and free their tensor memory), and with the
default bound restored the same handle must run the layer to a result that
matches the oracle.  The second case is large enough for f1 to run on CTA pairs
(the leader's bounded waits give up; the loaders then wait, within their own
bound, for the stages the products never consumed)."""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_inputs, oracle_params, rel_err
from helpers import oracle_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("lengths,d,H", [([100, 150, 6], 256, 2), ([700, 600], 1024, 8)])
def test_expired_waits_report_a_timeout_and_the_handle_recovers(lengths, d, H):
    batch = wl.make_custom_batch(lengths, d, H, seed=77, weight_scale=0.05 * (256 / d) ** 0.5,
                                 rab_scale=0.5)
    cfg = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16,
                           n_norm=1024, pos_buckets=129, pos_clamp=128, time_buckets=128,
                           time_log_div=0.301, ln_eps=1e-5, max_tokens=batch.total_tokens,
                           max_users=batch.num_users)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, "bf16", "bf16", "cuda:0")
    out = torch.empty_like(db.x)
    hstu.hstu_set_wait_limit(h.h, 1)
    h.forward(db, out, hstu.HSTU_MASK_CAUSAL)
    torch.cuda.synchronize()
    bits = h.device_error()
    assert bits & hstu.HSTU_DEVERR_TIMEOUT
    assert h.device_error() == 0           # reading the word cleared it
    hstu.hstu_set_wait_limit(h.h, 0)        # the default bound
    out.fill_(float("nan"))
    h.forward(db, out, hstu.HSTU_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert h.device_error() == 0
    y = out.double().cpu().numpy()
    h.close()
    ref = oracle.hstu_layer(oracle_inputs(batch, "bf16"), batch.seq_offsets, batch.timestamps,
                            batch.num_candidates, oracle_params(batch.layers[0], "bf16"),
                            oracle_cfg(d, H, n_norm=1024))
    assert rel_err(y, ref["Y"]) <= 2e-2
