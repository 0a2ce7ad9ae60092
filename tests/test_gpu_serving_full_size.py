"""GPU: M-FALCON serving against the history cache at the benchmark's full size
(8 users x (2048 history + 1024 candidates), d 512 = 8 heads x 64, micro-batches
of 256 candidates per user: the calls `bench.py --workload 4 --serve` times),
checked on sampled outputs.

The histories are prefilled once and every candidate is scored in four calls.
The candidates of users 0 and 5 are compared, element by element, with the
oracle's M-FALCON layer on that user alone ([history ; candidates], 3,072
tokens): a user's outputs depend on its own rows only, and a candidate sees
its user's history and itself, whichever call it comes in.  Bound: the bf16
one of the small cached-candidate cases, max-abs <= 2e-2 RMS + 2^-6 |ref|.
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_params
from helpers import cfg_for_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _pad_pair(n):
    return (n + 255) // 256 * 256


def test_serving_full_size_sampled():
    w = wl.WORKLOADS[4]
    batch = wl.make_batch(w, num_layers=1)
    B = batch.num_users
    n_c = [int(c) for c in batch.num_candidates]
    n_h = [int(n) - c for n, c in zip(batch.lengths, n_c)]
    offs = [int(o) for o in batch.seq_offsets]
    assert B == 8 and n_h == [2048] * B and n_c == [1024] * B
    bm = w.micro_batch
    hist = np.concatenate([np.arange(offs[b], offs[b] + n_h[b]) for b in range(B)]).astype(np.int64)
    T_h = len(hist)
    calls = []   # per call: (packed rows, counts)
    for k in range(max((c + bm - 1) // bm for c in n_c)):
        counts = [max(0, min(bm, c - k * bm)) for c in n_c]
        rows = np.concatenate([np.arange(offs[b] + n_h[b] + k * bm, offs[b] + n_h[b] + k * bm + counts[b])
                               for b in range(B)]).astype(np.int64)
        calls.append((rows, counts))
    max_cand_rows = max(sum(_pad_pair(c) for c in counts) for _, counts in calls)
    dev = torch.device("cuda", 0)
    cfg = runtime.config_for(w, max(_pad_pair(T_h) + max_cand_rows, batch.total_tokens), B)
    handle = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, w.storage, w.compute, dev)
    structs = [l.struct() for l in db.layers]
    stream = torch.cuda.current_stream(dev)
    hidx = torch.from_numpy(hist).to(dev)
    x_h = db.x[hidx].contiguous()
    ts_h = db.timestamps[hidx].contiguous()
    off_h = torch.from_numpy(wl.offsets_from_lengths(np.asarray(n_h)).astype(np.int32)).to(dev)
    y_h = torch.empty_like(x_h)
    cache = hstu.hstu_cache_create(handle.h, len(structs), T_h, max_cand_rows)
    hstu.hstu_cache_prefill(handle.h, cache, x_h, T_h, off_h, B, ts_h, structs, y_h, stream)
    y = torch.empty_like(db.x)   # candidate outputs at their packed rows
    for rows, counts in calls:
        ridx = torch.from_numpy(rows).to(dev)
        yc = torch.empty((len(rows), w.d_model), dtype=db.x.dtype, device=dev)
        hstu.hstu_cache_score(handle.h, cache, db.x[ridx].contiguous(), counts,
                              db.timestamps[ridx].contiguous(), structs, yc, stream)
        y[ridx] = yc
    torch.cuda.synchronize()
    assert handle.device_error() == 0
    hstu.hstu_cache_destroy(cache)
    handle.close()

    ocfg = cfg_for_workload(w)
    params = oracle_params(batch.layers[0], w.compute)
    X = wl.round_to_storage(batch.x, w.storage).astype(np.float64)
    for b in (0, 5):
        lo, hi = offs[b], offs[b + 1]
        ref = oracle.hstu_layer(X[lo:hi], np.array([0, hi - lo]), batch.timestamps[lo:hi],
                                np.array([n_c[b]], dtype=np.int32), params, ocfg)["Y"][n_h[b]:]
        got = y[lo + n_h[b]:hi].double().cpu().numpy()
        r = float(np.sqrt(np.mean(ref * ref)))
        err = np.abs(got - ref)
        assert np.all(err <= 2e-2 * r + 2.0 ** -6 * np.abs(ref)), (b, float(err.max()), r)
