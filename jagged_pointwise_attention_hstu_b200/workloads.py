"""Seeded synthetic inputs for the jagged HSTU layer forward.

This module only draws random inputs: sequence lengths, timestamps, the
Stochastic-Length subsampling of a batch, token features and random-init layer
parameters.  It holds none of the layer's arithmetic (no projection, SiLU,
bucketing, attention or normalisation), so both the CUDA path and the fp64
oracle can consume the same arrays without sharing any computation.

Workload shapes follow the pages' own workloads:

* jagged per-user sequences of interleaved item/action tokens ordered by
  timestamp ("Actions Speak Louder than Words", blog "Generative
  Recommendation 16: HSTU", section on turning heterogeneous features into a
  timeline; aitrending "How Generative Recommenders Are Redefining RecSys at
  Scale", Technical Details);
* the largest configuration: length 8192, embedding 1024, 24 layers (blog
  "Generative Recommendation 16: HSTU", section on what the experiments show);
* Stochastic Length with alpha = 1.6 mapping length 4096 mostly to 776
  (ltzyclt blog on HSTU, section 5.1; blog "Generative Recommendation 16",
  item 2 of the three extra pieces);
* M-FALCON candidates micro-batched after a user's history (ltzyclt blog,
  section 5.2).

Numeric constants of each workload (length laws, seeds, table sizes, weight
scales) are fixed by the layer configuration, not by the pages.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

SEED_BASE = 20261202

# Stochastic Length constants: keep the whole sequence with probability
# N_c^alpha / n^2, else keep an ordered random subset of N_c positions.
SL_NC = 776
SL_ALPHA = 1.6

ITEM_VOCAB = 1 << 14
ACTION_VOCAB = 8


@dataclass(frozen=True)
class Workload:
    """Static description of one synthetic workload."""
    name: str
    index: int
    num_users: int
    d_model: int
    num_heads: int
    head_dim: int
    num_layers: int
    storage: str            # dtype of X / Y in HBM: "fp32" or "bf16"
    compute: str            # "fp32" (SIMT path) or "bf16" (tensor-core path)
    pos_buckets: int
    pos_clamp: int
    time_buckets: int
    time_log_div: float
    n_norm: int             # > 0 fixed; <= 0 means "max length in the batch"
    mask: str               # "causal" or "mfalcon"
    lengths: str            # length law, see draw_lengths
    features: str           # "normal_0.02", "normal_1", "interleaved"
    history_len: int = 0    # M-FALCON only
    num_candidates: int = 0  # M-FALCON only
    micro_batch: int = 0    # M-FALCON b_m (only sets n_norm)
    stochastic_length: bool = False
    ln_eps: float = 1e-5

    @property
    def tokens_hint(self) -> str:
        return {0: "~288", 1: "~7.6k", 2: "~11.7k", 3: "65536", 4: "24576"}[self.index]


WORKLOADS = {
    0: Workload("single layer fp32, 4 users U[16,128], d64 2x32, causal", 0,
                num_users=4, d_model=64, num_heads=2, head_dim=32, num_layers=1,
                storage="fp32", compute="fp32", pos_buckets=129, pos_clamp=128,
                time_buckets=128, time_log_div=0.301, n_norm=0, mask="causal",
                lengths="uniform_16_128", features="normal_0.02"),
    1: Workload("single layer bf16, 32 users Zipf(1.2) in [32,1024], d256 4x64, causal", 1,
                num_users=32, d_model=256, num_heads=4, head_dim=64, num_layers=1,
                storage="bf16", compute="bf16", pos_buckets=129, pos_clamp=128,
                time_buckets=128, time_log_div=0.301, n_norm=1024, mask="causal",
                lengths="zipf_1.2_32_1024", features="interleaved"),
    2: Workload("single layer bf16, 16 users lognormal + Stochastic Length, d512 8x64, causal", 2,
                num_users=16, d_model=512, num_heads=8, head_dim=64, num_layers=1,
                storage="bf16", compute="bf16", pos_buckets=129, pos_clamp=128,
                time_buckets=128, time_log_div=0.301, n_norm=4096, mask="causal",
                lengths="lognormal_1500_0.8_4096", features="normal_1",
                stochastic_length=True),
    3: Workload("24-layer stack bf16, 8 users x 8192, d1024 8x128, causal", 3,
                num_users=8, d_model=1024, num_heads=8, head_dim=128, num_layers=24,
                storage="fp32", compute="bf16", pos_buckets=8193, pos_clamp=1024,
                time_buckets=128, time_log_div=0.301, n_norm=8192, mask="causal",
                lengths="fixed_8192", features="normal_1"),
    4: Workload("M-FALCON single layer bf16, 8 users x (2048 history + 1024 candidates), d512 8x64", 4,
                num_users=8, d_model=512, num_heads=8, head_dim=64, num_layers=1,
                storage="bf16", compute="bf16", pos_buckets=129, pos_clamp=128,
                time_buckets=128, time_log_div=0.301, n_norm=2048 + 256, mask="mfalcon",
                lengths="mfalcon", features="interleaved",
                history_len=2048, num_candidates=1024, micro_batch=256),
}


@dataclass
class LayerParams:
    """Random-init parameters of one HSTU layer (fp32 master copies).

    w1: [4d, d] (output-major, like a Linear weight), b1: [4d]
    w2: [d, d], b2: [d]
    rab_pos: [pos_buckets], rab_time: [time_buckets]
    ln_gamma, ln_beta: [d]
    """
    w1: np.ndarray
    b1: np.ndarray
    w2: np.ndarray
    b2: np.ndarray
    rab_pos: np.ndarray
    rab_time: np.ndarray
    ln_gamma: np.ndarray
    ln_beta: np.ndarray


@dataclass
class Batch:
    """One jagged batch: per-user sequences packed back to back, no padding."""
    lengths: np.ndarray          # int64 [B]
    seq_offsets: np.ndarray      # int32 [B+1], seq_offsets[0] = 0, [B] = T
    timestamps: np.ndarray       # int64 [T], non-decreasing inside each user
    num_candidates: np.ndarray   # int32 [B] (zeros for causal workloads)
    x: np.ndarray                # float32 [T, d]
    layers: List[LayerParams] = field(default_factory=list)

    @property
    def total_tokens(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def num_users(self) -> int:
        return int(self.lengths.shape[0])


def _streams(index: int, seed_offset: int = 0):
    ss = np.random.SeedSequence(SEED_BASE + index + 1000 * seed_offset)
    kids = ss.spawn(6)
    return {name: kid for name, kid in
            zip(("lengths", "sl", "timestamps", "features", "weights", "misc"), kids)}


def draw_lengths(law: str, num_users: int, rng: np.random.Generator) -> np.ndarray:
    """Per-user sequence lengths (int64) for the named length law."""
    if law == "uniform_16_128":
        return rng.integers(16, 128, size=num_users, endpoint=True).astype(np.int64)
    if law == "zipf_1.2_32_1024":
        # Zipf(a=1.2) restricted to its support inside [32, 1024] (a truncated
        # pmf, sampled exactly by inverse CDF on the finite support).
        k = np.arange(32, 1025, dtype=np.float64)
        pmf = k ** -1.2
        pmf /= pmf.sum()
        return rng.choice(np.arange(32, 1025), size=num_users, p=pmf).astype(np.int64)
    if law == "lognormal_1500_0.8_4096":
        raw = rng.lognormal(mean=np.log(1500.0), sigma=0.8, size=num_users)
        return np.clip(np.rint(raw), 1, 4096).astype(np.int64)
    if law == "fixed_8192":
        return np.full(num_users, 8192, dtype=np.int64)
    raise ValueError(f"unknown length law {law!r}")


def sl_keep_full_probability(n: np.ndarray) -> np.ndarray:
    """Probability that Stochastic Length keeps a length-n sequence whole."""
    n = np.asarray(n, dtype=np.float64)
    return np.minimum(1.0, SL_NC ** SL_ALPHA / np.maximum(n, 1.0) ** 2)


def stochastic_length_positions(n: int, rng: np.random.Generator) -> np.ndarray:
    """Kept positions (sorted) of one length-n sequence under Stochastic Length.

    Whole sequence with probability min(1, N_c^alpha / n^2); otherwise an
    ordered uniform subset of N_c positions.  A sequence no longer than N_c is
    always kept whole (a subset of N_c positions cannot be drawn from it).
    """
    u = rng.random()
    if u < sl_keep_full_probability(n) or n <= SL_NC:
        return np.arange(n, dtype=np.int64)
    return np.sort(rng.choice(n, size=SL_NC, replace=False)).astype(np.int64)


def draw_timestamps(n: int, rng: np.random.Generator) -> np.ndarray:
    """Integer-second timestamps: an epoch base plus cumulative Exp(3600 s) gaps."""
    base = 1_700_000_000 + int(rng.integers(0, 86_400 * 365))
    gaps = rng.exponential(3600.0, size=n)
    return (base + np.floor(np.cumsum(gaps))).astype(np.int64)


def _features_for_users(kind: str, lengths: np.ndarray, d: int, rng: np.random.Generator,
                        candidate_counts: Optional[np.ndarray] = None) -> np.ndarray:
    total = int(lengths.sum())
    if kind == "normal_0.02":
        return rng.normal(0.0, 0.02, size=(total, d)).astype(np.float32)
    if kind == "normal_1":
        return rng.normal(0.0, 1.0, size=(total, d)).astype(np.float32)
    if kind != "interleaved":
        raise ValueError(kind)
    emb_item = rng.normal(0.0, 1.0, size=(ITEM_VOCAB, d)).astype(np.float32)
    emb_action = rng.normal(0.0, 1.0, size=(ACTION_VOCAB, d)).astype(np.float32)
    emb_type = rng.normal(0.0, 1.0, size=(2, d)).astype(np.float32)
    # Zipf-like item popularity over a finite vocabulary.
    ranks = np.arange(1, ITEM_VOCAB + 1, dtype=np.float64)
    item_p = ranks ** -1.1
    item_p /= item_p.sum()
    out = np.empty((total, d), dtype=np.float32)
    row = 0
    for b, n in enumerate(lengths):
        n = int(n)
        n_c = 0 if candidate_counts is None else int(candidate_counts[b])
        n_h = n - n_c
        t = np.arange(n)
        is_action = (t % 2 == 1) & (t < n_h)        # candidates are item tokens
        ids_item = rng.choice(ITEM_VOCAB, size=n, p=item_p)
        ids_action = rng.integers(0, ACTION_VOCAB, size=n)
        tok = np.where(is_action[:, None], emb_action[ids_action], emb_item[ids_item])
        typ = emb_type[is_action.astype(np.int64)]
        out[row:row + n] = (tok + typ) / np.float32(np.sqrt(2.0))
        row += n
    return out


def random_layer(w: Workload, rng: np.random.Generator, scale: float = 0.02) -> LayerParams:
    d = w.d_model
    return LayerParams(
        w1=rng.normal(0.0, scale, size=(4 * d, d)).astype(np.float32),
        b1=rng.normal(0.0, scale, size=(4 * d,)).astype(np.float32),
        w2=rng.normal(0.0, scale, size=(d, d)).astype(np.float32),
        b2=rng.normal(0.0, scale, size=(d,)).astype(np.float32),
        rab_pos=rng.normal(0.0, scale, size=(w.pos_buckets,)).astype(np.float32),
        rab_time=rng.normal(0.0, scale, size=(w.time_buckets,)).astype(np.float32),
        ln_gamma=np.ones((d,), dtype=np.float32),
        ln_beta=np.zeros((d,), dtype=np.float32),
    )


def offsets_from_lengths(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    if off[-1] >= 2 ** 31:
        raise ValueError("total tokens must stay below 2^31")
    return off.astype(np.int32)


def make_batch(w: Workload, *, num_layers: Optional[int] = None, seed_offset: int = 0,
               num_users: Optional[int] = None, max_len: Optional[int] = None) -> Batch:
    """Draw the seeded batch of workload ``w``.

    ``num_layers`` limits how many layers' parameters are drawn (the first
    ones; later layers keep their own streams).  ``num_users`` keeps the first
    users; ``max_len`` truncates every user to its first ``max_len`` tokens
    (a causal prefix: the same draws, cut short).
    """
    st = _streams(w.index, seed_offset)
    rl = np.random.default_rng(st["lengths"])
    B = w.num_users
    if w.lengths == "mfalcon":
        lengths = np.full(B, w.history_len + w.num_candidates, dtype=np.int64)
        ncand = np.full(B, w.num_candidates, dtype=np.int32)
    else:
        lengths = draw_lengths(w.lengths, B, rl)
        ncand = np.zeros(B, dtype=np.int32)

    rt = np.random.default_rng(st["timestamps"])
    rsl = np.random.default_rng(st["sl"])
    ts_users = []
    for b in range(B):
        n = int(lengths[b])
        if w.lengths == "mfalcon":
            hist = draw_timestamps(w.history_len, rt)
            cand = np.full(w.num_candidates, hist[-1], dtype=np.int64)
            ts_users.append(np.concatenate([hist, cand]))
            continue
        ts = draw_timestamps(n, rt)
        if w.stochastic_length:
            keep = stochastic_length_positions(n, rsl)
            ts = ts[keep]
            lengths[b] = keep.shape[0]
        ts_users.append(ts)

    if num_users is not None:
        lengths, ncand, ts_users = lengths[:num_users], ncand[:num_users], ts_users[:num_users]
    if max_len is not None:
        if w.mask == "mfalcon":
            raise ValueError("prefix truncation is defined for causal workloads only")
        lengths = np.minimum(lengths, max_len)
        ts_users = [t[:max_len] for t in ts_users]

    rf = np.random.default_rng(st["features"])
    if w.features == "interleaved":
        x = _features_for_users("interleaved", lengths, w.d_model, rf, ncand)
    else:
        # Draw the full-length rows user by user so that a prefix batch holds
        # exactly the leading rows of the full batch.
        full_lengths = draw_lengths(w.lengths, w.num_users,
                                    np.random.default_rng(st["lengths"])) \
            if w.lengths != "mfalcon" else None
        rows = []
        for b in range(len(lengths)):
            n_full = int(full_lengths[b]) if (full_lengths is not None and not w.stochastic_length) \
                else int(lengths[b])
            scale = 0.02 if w.features == "normal_0.02" else 1.0
            blk = rf.normal(0.0, scale, size=(n_full, w.d_model)).astype(np.float32)
            rows.append(blk[:int(lengths[b])])
        x = np.concatenate(rows, axis=0) if rows else np.zeros((0, w.d_model), np.float32)

    nl = w.num_layers if num_layers is None else num_layers
    layer_seeds = st["weights"].spawn(w.num_layers)
    layers = [random_layer(w, np.random.default_rng(layer_seeds[l])) for l in range(nl)]

    ts = np.concatenate(ts_users) if ts_users else np.zeros((0,), np.int64)
    return Batch(lengths=lengths.astype(np.int64), seq_offsets=offsets_from_lengths(lengths),
                 timestamps=ts.astype(np.int64), num_candidates=ncand.astype(np.int32),
                 x=x, layers=layers)


def make_custom_batch(lengths, d_model: int, num_heads: int, *, seed: int,
                      num_candidates=None, pos_buckets: int = 129, time_buckets: int = 128,
                      feature_scale: float = 1.0, weight_scale: float = 0.02,
                      rab_scale: Optional[float] = None, random_affine: bool = False,
                      num_layers: int = 1, timestamp_gap: float = 3600.0) -> Batch:
    """Small batch with explicit per-user lengths, for edge-case tests.

    ``rab_scale`` (default: ``weight_scale``) sets the spread of both bias
    tables; a large value makes every bucket index matter for the output.
    ``random_affine`` draws LayerNorm gamma/beta instead of 1/0.
    """
    rng = np.random.default_rng(np.random.SeedSequence(SEED_BASE + 7919 * (seed + 1)))
    lengths = np.asarray(lengths, dtype=np.int64)
    B = lengths.shape[0]
    ncand = np.zeros(B, np.int32) if num_candidates is None else np.asarray(num_candidates, np.int32)
    ts = []
    for b in range(B):
        n = int(lengths[b])
        n_h = n - int(ncand[b])
        base = 1_700_000_000 + int(rng.integers(0, 10_000_000))
        hist = (base + np.floor(np.cumsum(rng.exponential(timestamp_gap, size=n_h)))).astype(np.int64)
        last = hist[-1] if n_h > 0 else np.int64(base)
        ts.append(np.concatenate([hist, np.full(n - n_h, last, np.int64)]))
    x = rng.normal(0.0, feature_scale, size=(int(lengths.sum()), d_model)).astype(np.float32)
    rs = weight_scale if rab_scale is None else rab_scale
    layers = []
    for _ in range(num_layers):
        d = d_model
        lp = LayerParams(
            w1=rng.normal(0.0, weight_scale, size=(4 * d, d)).astype(np.float32),
            b1=rng.normal(0.0, weight_scale, size=(4 * d,)).astype(np.float32),
            w2=rng.normal(0.0, weight_scale, size=(d, d)).astype(np.float32),
            b2=rng.normal(0.0, weight_scale, size=(d,)).astype(np.float32),
            rab_pos=rng.normal(0.0, rs, size=(pos_buckets,)).astype(np.float32),
            rab_time=rng.normal(0.0, rs, size=(time_buckets,)).astype(np.float32),
            ln_gamma=(rng.normal(1.0, 0.1, size=(d,)) if random_affine else np.ones(d)).astype(np.float32),
            ln_beta=(rng.normal(0.0, 0.1, size=(d,)) if random_affine else np.zeros(d)).astype(np.float32),
        )
        layers.append(lp)
    return Batch(lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
                 timestamps=np.concatenate(ts) if ts else np.zeros((0,), np.int64),
                 num_candidates=ncand, x=x, layers=layers)


def round_to_storage(a: np.ndarray, storage: str) -> np.ndarray:
    """Values exactly as they sit in HBM for ``storage`` ("fp32" or "bf16"),
    returned as float32 (bf16 by round-to-nearest-even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if storage == "fp32":
        return a.copy()
    if storage != "bf16":
        raise ValueError(storage)
    bits = a.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the upper 16 bits; NaN/Inf do not occur here
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bf16 encodings of ``a`` (round-to-nearest-even)."""
    r = round_to_storage(a, "bf16")
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def with_layers(batch: Batch, layers: List[LayerParams]) -> Batch:
    return dataclasses.replace(batch, layers=layers)
