"""GPU: M-FALCON scoring against a history cache, through the C ABI.

A cache keeps every layer's SiLU(f1(.)) of the users' histories; each scoring
call runs the stack on one micro-batch of candidates only.  The candidates'
outputs must be those of the whole M-FALCON batch [history ; candidates] per
user (ltzyclt blog, section 5.2: a candidate sees the history and itself),
which the oracle computes directly on that packed batch.

Tolerances against the oracle:
  Y max-abs <= 2e-2 x RMS(Y), the layer tolerance of the bf16 path, with an
  fp32 residual stream.  With a bf16 stream the oracle rounds its stream to
  bf16 between the layers as the stored layer inputs are, and leaves its last
  output unrounded; since the two sides round slightly different values, the
  stored layer input may sit one bf16 ulp (<= 2^-7 |x|) from the oracle's, and
  the output's own rounding adds half an ulp: per element
  |err| <= 2e-2 x RMS(Y) + 2^-6 |Y|  (1.5 x 2^-7 |x|, with slack for |x| > |Y|).
  With an fp32 residual stream also the layers' total update Y - X:
  max-abs <= 5e-2 x RMS(update).  Every bf16 rounding of the path (the GEMM
  operands X and G, U|V|Q|K, P: 2^-9 relative each, about a dozen per layer,
  two layers) reaches the update, which the oracle computes unrounded:
  25 x 2^-9 ~ 5e-2.
Bit for bit:
  prefill                the causal stack on the histories (the same kernels
                         on the same rows)
  micro-batches          a candidate row reads only its own inputs and its
                         user's cached history; every query tile of the
                         candidate block holds one user's rows, which share
                         their row facts and timestamp, so every warp takes
                         the same path whatever the partition into calls
  plain M-FALCON stack   with every history and candidate count a multiple of
  (aligned layout)       256, the packed batch [history ; candidates] puts
                         every user's rows at the same offsets inside their
                         query-tile pairs as the cache does, so each candidate
                         row visits the same keys in the same tiles in the
                         same order: the same arithmetic.  (Ragged layouts
                         split a history's keys into tiles differently, which
                         changes only the order of fp32 sums.)
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import oracle_params, rel_err
from helpers import oracle_cfg

pytestmark = pytest.mark.gpu

N_H = [300, 0, 700, 129, 256]   # history lengths: empty, tile-aligned and ragged
N_C = [40, 256, 3, 300, 0]      # candidates: one pair, ragged, none
N_NORM = 1024
D, LAYERS = 256, 2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _pad(n):
    return (n + 255) // 256 * 256


def _batch(H, seed, n_h, n_c):
    lengths = [h + c for h, c in zip(n_h, n_c)]
    return wl.make_custom_batch(lengths, D, H, seed=seed, num_candidates=n_c, weight_scale=0.05,
                                rab_scale=1.0, random_affine=True, num_layers=LAYERS,
                                timestamp_gap=900.0)


def _split(batch, n_h, n_c):
    """Row indices of the histories and of the candidates in the packed batch."""
    hist, cand = [], []
    for b, (h, c) in enumerate(zip(n_h, n_c)):
        s = int(batch.seq_offsets[b])
        hist.extend(range(s, s + h))
        cand.extend(range(s + h, s + h + c))
    return np.asarray(hist, np.int64), np.asarray(cand, np.int64)


def _oracle_candidates(batch, storage, H, cand_rows):
    """The oracle's M-FALCON stack on the packed batch; candidate rows of Y and X."""
    cfg = oracle_cfg(D, H, n_norm=N_NORM, mask="mfalcon")
    X0 = wl.round_to_storage(batch.x, storage).astype(np.float64)
    X = X0
    for l, lp in enumerate(batch.layers):
        Y = oracle.hstu_layer(X, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                              oracle_params(lp, "bf16"), cfg)["Y"]
        last = l + 1 == len(batch.layers)
        X = wl.round_to_storage(Y.astype(np.float32), storage).astype(np.float64) \
            if storage == "bf16" and not last else Y
    return X[cand_rows], X0[cand_rows]


class _Setup:
    def __init__(self, storage, H, seed, n_h=N_H, n_c=N_C):
        self.n_h, self.n_c = list(n_h), list(n_c)
        self.batch = _batch(H, seed, self.n_h, self.n_c)
        self.hist, self.cand = _split(self.batch, self.n_h, self.n_c)
        self.T_h = len(self.hist)
        self.storage = storage
        cand_rows = sum(_pad(c) for c in self.n_c)
        rows_cap = _pad(self.T_h) + cand_rows
        cfg = hstu.make_config(
            D, H, io_dtype=hstu.HSTU_DTYPE_BF16 if storage == "bf16" else hstu.HSTU_DTYPE_FP32,
            compute_dtype=hstu.HSTU_DTYPE_BF16, n_norm=N_NORM, pos_buckets=129, pos_clamp=128,
            time_buckets=128, time_log_div=0.301, ln_eps=1e-5,
            max_tokens=max(rows_cap, self.batch.total_tokens), max_users=len(self.n_h))
        self.handle = runtime.Handle(cfg, 0)
        self.layers = runtime.device_layers(self.batch, "bf16", "cuda:0")
        self.structs = [l.struct() for l in self.layers]
        dt = torch.bfloat16 if storage == "bf16" else torch.float32
        dev = "cuda:0"
        self.x = torch.from_numpy(self.batch.x).to(device=dev, dtype=dt)
        self.ts = torch.from_numpy(self.batch.timestamps).to(dev)
        self.x_h = self.x[torch.from_numpy(self.hist).to(dev)].contiguous()
        self.ts_h = self.ts[torch.from_numpy(self.hist).to(dev)].contiguous()
        self.off_h = torch.from_numpy(
            wl.offsets_from_lengths(np.asarray(self.n_h)).astype(np.int32)).to(dev)
        self.cache = hstu.hstu_cache_create(self.handle.h, LAYERS, self.T_h, cand_rows)

    def prefill(self):
        y = torch.empty_like(self.x_h)
        hstu.hstu_cache_prefill(self.handle.h, self.cache, self.x_h, self.T_h, self.off_h,
                                len(self.n_h), self.ts_h, self.structs, y,
                                torch.cuda.current_stream())
        return y

    def score(self, take):
        """Scores, per user b, the candidates take[b] (local indices); returns Y rows."""
        rows = np.concatenate([np.asarray(self.cand_of(b)[t], np.int64)
                               for b, t in enumerate(take)])
        ridx = torch.from_numpy(rows).to("cuda:0")
        x_c = self.x[ridx].contiguous()
        ts_c = self.ts[ridx].contiguous()
        y = torch.empty_like(x_c)
        hstu.hstu_cache_score(self.handle.h, self.cache, x_c, [len(t) for t in take], ts_c,
                              self.structs, y, torch.cuda.current_stream())
        return y

    def cand_of(self, b):
        s = int(self.batch.seq_offsets[b]) + self.n_h[b]
        return np.arange(s, s + self.n_c[b])

    def close(self):
        torch.cuda.synchronize()
        assert self.handle.device_error() == 0
        hstu.hstu_cache_destroy(self.cache)
        self.handle.close()


@pytest.mark.parametrize("storage,H", [("fp32", 4), ("bf16", 2)])
def test_cached_candidates_match_the_oracle(storage, H):
    s = _Setup(storage, H, seed=31 + H)
    s.prefill()
    y = s.score([np.arange(c) for c in s.n_c]).double().cpu().numpy()
    ref, x0 = _oracle_candidates(s.batch, storage, H, s.cand)
    s.close()
    assert y.shape == ref.shape
    if storage == "fp32":
        assert rel_err(y, ref) <= 2e-2
        assert rel_err(y - x0, ref - x0) <= 5e-2
    else:
        r = np.sqrt(np.mean(ref * ref))
        assert np.all(np.abs(y - ref) <= 2e-2 * r + 2.0 ** -6 * np.abs(ref))


@pytest.mark.parametrize("storage", ["fp32", "bf16"])
def test_aligned_cached_candidates_equal_the_plain_stack(storage):
    s = _Setup(storage, 4, seed=17, n_h=[256, 512, 0], n_c=[256, 256, 512])
    s.prefill()
    y = s.score([np.arange(c) for c in s.n_c])
    db = runtime.DeviceBatch(
        x=s.x, seq_offsets=torch.from_numpy(s.batch.seq_offsets.astype(np.int32)).cuda(),
        timestamps=s.ts, num_candidates=torch.from_numpy(s.batch.num_candidates).cuda(),
        layers=s.layers, total_tokens=s.batch.total_tokens, num_users=len(s.n_h))
    plain = torch.empty_like(s.x)
    s.handle.forward(db, plain, hstu.HSTU_MASK_MFALCON)
    s.close()
    assert torch.equal(y, plain[torch.from_numpy(s.cand).cuda()])


def test_prefill_equals_the_causal_stack_and_micro_batches_are_exact():
    s = _Setup("bf16", 4, seed=5)
    y_h = s.prefill()
    # the plain causal stack on the histories, same handle
    db = runtime.DeviceBatch(x=s.x_h, seq_offsets=s.off_h, timestamps=s.ts_h,
                             num_candidates=torch.zeros(len(N_H), dtype=torch.int32, device="cuda:0"),
                             layers=s.layers, total_tokens=s.T_h, num_users=len(N_H))
    ref = torch.empty_like(s.x_h)
    s.handle.forward(db, ref, hstu.HSTU_MASK_CAUSAL)
    assert torch.equal(y_h, ref)
    # all candidates in one call, then in two calls with a different split per user
    full = s.score([np.arange(c) for c in N_C])
    rng = np.random.default_rng(3)
    first, second = [], []
    for c in N_C:
        perm = rng.permutation(c)
        k = int(rng.integers(0, c + 1))
        first.append(np.sort(perm[:k]))
        second.append(np.sort(perm[k:]))
    y1 = s.score(first)
    y2 = s.score(second)
    # reassemble by packed candidate index
    pos = np.concatenate([[0], np.cumsum(N_C)])
    got = torch.empty_like(full)
    i1 = np.concatenate([pos[b] + first[b] for b in range(len(N_C))]).astype(np.int64)
    i2 = np.concatenate([pos[b] + second[b] for b in range(len(N_C))]).astype(np.int64)
    got[torch.from_numpy(i1).cuda()] = y1
    got[torch.from_numpy(i2).cuda()] = y2
    assert torch.equal(got, full)
    s.close()


def test_cache_argument_errors():
    s = _Setup("bf16", 4, seed=8)
    take = [np.arange(c) for c in N_C]
    with pytest.raises(hstu.HstuError) as e:            # no history yet
        s.score(take)
    assert e.value.status == hstu.HSTU_ERR_INVALID_ARG
    s.prefill()
    counts = list(N_C)
    counts[0] += 256                                    # one more pair than the capacity
    with pytest.raises(hstu.HstuError) as e:
        hstu.hstu_cache_score(s.handle.h, s.cache, s.x_h, counts, s.ts_h, s.structs, s.x_h, None)
    assert e.value.status == hstu.HSTU_ERR_WORKSPACE
    with pytest.raises(hstu.HstuError) as e:            # layer count differs from the cache's
        hstu.hstu_cache_score(s.handle.h, s.cache, s.x_h, [1] * len(N_H), s.ts_h,
                              s.structs[:1], s.x_h, None)
    assert e.value.status == hstu.HSTU_ERR_INVALID_ARG
    # no candidates at all: nothing to do
    hstu.hstu_cache_score(s.handle.h, s.cache, None, [0] * len(N_H), None, s.structs, None, None)
    with pytest.raises(hstu.HstuError) as e:            # the cache would not fit the workspace
        hstu.hstu_cache_create(s.handle.h, LAYERS, 1 << 20, 256)
    assert e.value.status == hstu.HSTU_ERR_WORKSPACE
    s.close()
    cfg = hstu.make_config(D, 4, io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16,
                           n_norm=0, pos_buckets=129, pos_clamp=128, time_buckets=128,
                           time_log_div=0.301, ln_eps=1e-5, max_tokens=4096, max_users=4)
    h = runtime.Handle(cfg, 0)
    with pytest.raises(hstu.HstuError) as e:            # n_norm from each call's lengths
        hstu.hstu_cache_create(h.h, 1, 1024, 256)
    assert e.value.status == hstu.HSTU_ERR_UNSUPPORTED
    h.close()
