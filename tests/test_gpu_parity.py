"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerances (inputs identical on both sides: the oracle receives the exact
values stored in HBM):
  fp32 path   Y max-abs <= 1e-4; intermediates <= 1e-5 x RMS (fp32 sums of
              <= 129 terms carry <= 129 * 2^-24 relative error).
  bf16 path   Y max-abs <= 2e-2 x RMS(Y).
              U,V,Q,K and G are stored in bf16 (half an ulp is 2^-9 of the
              value): per element |err| <= 2^-8 |ref| + 1e-3 RMS(ref).
              The attention output O is compared with the oracle's equation
              (2) evaluated on the GPU's own U,V,Q,K, so only the kernel's own
              rounding remains (P in bf16, tanh-based SiLU within 2^-10,
              fp32 accumulation): per element
              |err| <= 2^-7 * sum_j |a_ij| |v_j| + 1e-6 RMS(O),
              the standard bound of a dot product with relative term errors.
Bucket indices and the mask are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_pointwise_attention_hstu_b200 import build, hstu, runtime
from jagged_pointwise_attention_hstu_b200 import workloads as wl

from gpu_common import gpu_run, oracle_inputs, oracle_params, rel_err, teacher_forced_attention
from helpers import cfg_for_workload, oracle_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    hstu.load()


# ------------------------------------------------------------ operand layouts

@pytest.mark.parametrize("mode,n,k", [(0, 128, 64), (0, 256, 128), (0, 64, 128),
                                      (1, 64, 128), (1, 128, 128), (2, 64, 128), (2, 128, 128)])
def test_umma_tile_layouts(mode, n, k):
    g = torch.Generator().manual_seed(mode * 1000 + n + k)
    A = torch.randn(128, k, generator=g).to(torch.bfloat16).cuda()
    if mode == 0:
        B = torch.randn(n, k, generator=g).to(torch.bfloat16).cuda()
        ref = A.float() @ B.float().T
    else:
        B = torch.randn(k, n, generator=g).to(torch.bfloat16).cuda()
        ref = A.float() @ B.float()
    C = torch.empty(128, n, dtype=torch.float32, device="cuda")
    hstu.hstu_debug_umma_tile(mode, A, B, C, n, k)
    torch.cuda.synchronize()
    err = (C - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), f"mode {mode}: max err {err}"


# ------------------------------------------------------------ workloads

def _check_layer(w, batch, res):
    cfg = cfg_for_workload(w)
    p = oracle_params(batch.layers[0], w.compute)
    X = oracle_inputs(batch, w.storage)
    ref = oracle.hstu_layer(X, batch.seq_offsets, batch.timestamps, batch.num_candidates, p, cfg)
    d = w.d_model
    assert res["error"] == 0
    if w.compute == "fp32":
        assert np.max(np.abs(res["Y"] - ref["Y"])) <= 1e-4
        uvqk = np.concatenate([ref["U"], ref["V"], ref["Q"], ref["K"]], axis=1)
        assert rel_err(res["UVQK"], uvqk) <= 1e-5
        assert rel_err(res["AV"], ref["O"]) <= 1e-5
        assert rel_err(res["G"], ref["G"]) <= 1e-4
        return ref
    # bf16 tensor-core path
    assert rel_err(res["Y"], ref["Y"]) <= 2e-2
    uvqk = np.concatenate([ref["U"], ref["V"], ref["Q"], ref["K"]], axis=1)
    if w.storage == "fp32":
        # an fp32 residual stream with bf16 operands: f1's GEMM reads bf16(X), so
        # its outputs are compared with f1 evaluated on that input (the residual
        # and everything checked above keep the exact fp32 X)
        Xb = oracle_inputs(batch, "bf16")
        uvqk = np.concatenate(oracle.f1_split(Xb, p["w1"], p["b1"], d), axis=1)
    r = np.sqrt(np.mean(uvqk ** 2))
    assert np.all(np.abs(res["UVQK"] - uvqk) <= 2.0 ** -8 * np.abs(uvqk) + 1e-3 * r)
    O_tf, O_abs = teacher_forced_attention(res["UVQK"], batch, cfg, p, with_abs=True)
    rO = np.sqrt(np.mean(O_tf ** 2)) if O_tf.size else 0.0
    assert np.all(np.abs(res["AV"] - O_tf) <= 2.0 ** -7 * O_abs + 1e-6 * rO)
    N_tf = oracle.layer_norm(res["AV"], p["ln_gamma"], p["ln_beta"], cfg.ln_eps)
    G_tf = N_tf * res["UVQK"][:, :d]
    rG = np.sqrt(np.mean(G_tf ** 2)) if G_tf.size else 0.0
    assert np.all(np.abs(res["G"] - G_tf) <= 2.0 ** -8 * np.abs(G_tf) + 1e-3 * rG)
    return ref


@pytest.mark.parametrize("idx", [0, 1, 2, 4])
def test_workload_parity(idx):
    w = wl.WORKLOADS[idx]
    batch = wl.make_batch(w)
    res = gpu_run(batch, w.storage, w.compute, d=w.d_model, H=w.num_heads, n_norm=w.n_norm,
                  mask=w.mask, pos_buckets=w.pos_buckets, pos_clamp=w.pos_clamp,
                  time_buckets=w.time_buckets, div=w.time_log_div, eps=w.ln_eps)
    _check_layer(w, batch, res)


def test_fp32_path_with_strong_attention():
    """fp32 layer whose output depends strongly on attention and on every bias bucket."""
    w = wl.WORKLOADS[0]
    batch = wl.make_custom_batch([1, 37, 128, 129, 0, 90], 64, 2, seed=21, weight_scale=0.25,
                                 rab_scale=1.0, random_affine=True, feature_scale=1.0,
                                 timestamp_gap=600.0)
    res = gpu_run(batch, "fp32", "fp32", d=64, H=2, n_norm=0, mask="causal")
    _check_layer(w, batch, res)


@pytest.mark.parametrize("lengths", [[1800, 1700, 1220], [1800, 1700, 1333]])
def test_fp32_residual_stream_ragged_pair_tiles(lengths):
    """fp32 residual stream, bf16 compute, d 1024 (c3's precision and width) at
    ragged token counts large enough for the CTA-pair GEMMs (f2 takes its
    residual by TMA): 4720 tokens leave the second CTA of the last 256-row tile
    wholly past T, 4833 partly."""
    d, H = 1024, 8
    batch = wl.make_custom_batch(lengths, d, H, seed=sum(lengths), weight_scale=0.03,
                                 rab_scale=1.0, random_affine=True, timestamp_gap=900.0)
    w = wl.Workload("fp32 residual, ragged", 98, num_users=len(lengths), d_model=d, num_heads=H,
                    head_dim=128, num_layers=1, storage="fp32", compute="bf16", pos_buckets=129,
                    pos_clamp=128, time_buckets=128, time_log_div=0.301, n_norm=2048,
                    mask="causal", lengths="custom", features="normal_1")
    res = gpu_run(batch, "fp32", "bf16", d=d, H=H, n_norm=2048, mask="causal")
    _check_layer(w, batch, res)


# ------------------------------------------------------------ edge cases

EDGE_LENGTHS = [
    [1],
    [127, 1, 128, 129],
    [0, 5, 0, 0, 300, 0],
    [255, 256, 257],
    [3, 700, 2, 2, 41],
]


@pytest.mark.parametrize("lengths", EDGE_LENGTHS)
@pytest.mark.parametrize("hd", [64, 128])
def test_edge_lengths_causal(lengths, hd):
    d = 256
    H = d // hd
    batch = wl.make_custom_batch(lengths, d, H, seed=sum(lengths) + hd, weight_scale=0.05,
                                 rab_scale=1.0, random_affine=True, timestamp_gap=900.0)
    w = wl.Workload("edge", 99, num_users=len(lengths), d_model=d, num_heads=H, head_dim=hd,
                    num_layers=1, storage="bf16", compute="bf16", pos_buckets=129, pos_clamp=128,
                    time_buckets=128, time_log_div=0.301, n_norm=512, mask="causal",
                    lengths="custom", features="normal_1")
    res = gpu_run(batch, "bf16", "bf16", d=d, H=H, n_norm=512, mask="causal")
    _check_layer(w, batch, res)


@pytest.mark.parametrize("lengths,ncand", [
    ([300, 140], [100, 140]),          # second user holds candidates only
    ([130, 5, 260], [2, 5, 129]),
    ([1, 129, 383], [1, 0, 255]),
])
def test_edge_lengths_mfalcon(lengths, ncand):
    d, H = 256, 4
    batch = wl.make_custom_batch(lengths, d, H, seed=7 * sum(lengths), num_candidates=ncand,
                                 weight_scale=0.05, rab_scale=1.0, random_affine=True,
                                 timestamp_gap=900.0)
    w = wl.Workload("edge-mf", 98, num_users=len(lengths), d_model=d, num_heads=H, head_dim=64,
                    num_layers=1, storage="bf16", compute="bf16", pos_buckets=129, pos_clamp=128,
                    time_buckets=128, time_log_div=0.301, n_norm=400, mask="mfalcon",
                    lengths="custom", features="normal_1")
    res = gpu_run(batch, "bf16", "bf16", d=d, H=H, n_norm=400, mask="mfalcon")
    _check_layer(w, batch, res)


def test_empty_batch_is_a_no_op():
    d, H = 256, 4
    batch = wl.make_custom_batch([0, 0], d, H, seed=1)
    cfg = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16,
                           n_norm=0, pos_buckets=129, pos_clamp=128, time_buckets=128,
                           time_log_div=0.301, ln_eps=1e-5, max_tokens=16, max_users=4)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, "bf16", "bf16", "cuda:0")
    out = torch.empty((0, d), dtype=torch.bfloat16, device="cuda:0")
    h.forward(db, out, hstu.HSTU_MASK_CAUSAL)
    assert h.device_error() == 0
    h.close()


# ------------------------------------------------------------ buckets bit for bit

@pytest.mark.parametrize("mask,lengths,ncand,clamp", [
    ("causal", [200, 1, 0, 333, 130], None, 128),
    ("mfalcon", [260, 70, 200], [60, 70, 1], 128),
    ("causal", [1500], None, 1024),
])
def test_attention_buckets_bit_exact(mask, lengths, ncand, clamp):
    d, H = 256, 2
    # mixed gaps: seconds to years, so that many time buckets are crossed
    batch = wl.make_custom_batch(lengths, d, H, seed=len(lengths), num_candidates=ncand,
                                 timestamp_gap=20000.0)
    rng = np.random.default_rng(4)
    offs = batch.seq_offsets
    ts = batch.timestamps.copy()
    for b in range(len(lengths)):
        lo, hi = int(offs[b]), int(offs[b + 1])
        nc = 0 if ncand is None else ncand[b]
        nh = (hi - lo) - nc
        gaps = np.exp(rng.uniform(0, 20, size=nh)).astype(np.int64)
        hist = 1_000 + np.cumsum(gaps)
        ts[lo:lo + nh] = hist
        ts[lo + nh:hi] = hist[-1] if nh > 0 else 1_000
    T = batch.total_tokens
    cfg = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16,
                           n_norm=0, pos_buckets=clamp + 1, pos_clamp=clamp, time_buckets=128,
                           time_log_div=0.301, ln_eps=1e-5, max_tokens=T, max_users=len(lengths))
    h = runtime.Handle(cfg, 0)
    offs_d = torch.from_numpy(offs.astype(np.int32)).cuda()
    ts_d = torch.from_numpy(ts).cuda()
    nc_d = torch.from_numpy(batch.num_candidates).cuda()
    pidx = torch.full((T, T), -1, dtype=torch.int32, device="cuda")
    tidx = torch.full((T, T), -1, dtype=torch.int32, device="cuda")
    vis = torch.full((T, T), 255, dtype=torch.uint8, device="cuda")
    mode = hstu.HSTU_MASK_MFALCON if mask == "mfalcon" else hstu.HSTU_MASK_CAUSAL
    hstu.hstu_debug_attention_buckets(h.h, T, offs_d, len(lengths), ts_d, mode, nc_d, pidx, tidx,
                                      vis)
    assert h.device_error() == 0
    h.close()
    pidx, tidx, vis = pidx.cpu().numpy(), tidx.cpu().numpy(), vis.cpu().numpy()
    ocfg = oracle_cfg(d, H, pos_clamp=clamp, mask=mask)
    want_vis = np.zeros((T, T), dtype=bool)
    for b in range(len(lengths)):
        lo, hi = int(offs[b]), int(offs[b + 1])
        n = hi - lo
        if n == 0:
            continue
        nc = 0 if ncand is None else ncand[b]
        v, rel = oracle.user_visibility(n, nc, mask)
        want_vis[lo:hi, lo:hi] = v
        p_or = oracle.position_bucket(rel, clamp)
        t_or = oracle.time_bucket(ts[lo:hi][:, None] - ts[lo:hi][None, :], 0.301, 128)
        blk = np.s_[lo:hi, lo:hi]
        assert np.array_equal(pidx[blk][v], p_or[v])
        assert np.array_equal(tidx[blk][v], t_or[v])
    # every visible pair was visited and flagged; nothing else is flagged visible
    assert np.array_equal(vis == 1, want_vis)
    assert len(np.unique(tidx[want_vis])) > 20


# ------------------------------------------------------------ errors, determinism

@pytest.mark.parametrize("kind,bit", [("ts", hstu.HSTU_DEVERR_TIMESTAMPS),
                                      ("offsets", hstu.HSTU_DEVERR_OFFSETS),
                                      ("cand", hstu.HSTU_DEVERR_CANDIDATES)])
def test_invalid_inputs_set_the_device_error_word(kind, bit):
    d, H = 256, 4
    lengths = [100, 50]
    batch = wl.make_custom_batch(lengths, d, H, seed=3, num_candidates=[10, 5])
    cfg = hstu.make_config(d, H, io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16,
                           n_norm=0, pos_buckets=129, pos_clamp=128, time_buckets=128,
                           time_log_div=0.301, ln_eps=1e-5, max_tokens=256, max_users=4)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, "bf16", "bf16", "cuda:0")
    if kind == "ts":
        db.timestamps[60] = db.timestamps[59] - 5
    elif kind == "offsets":
        db.seq_offsets[1] = 160         # beyond T, and non-monotone
    else:
        db.num_candidates[1] = 51
    out = torch.empty_like(db.x)
    h.forward(db, out, hstu.HSTU_MASK_MFALCON)
    bits = h.device_error()
    assert bits & bit
    # the handle stays usable after the error
    db2 = runtime.to_device(batch, "bf16", "bf16", "cuda:0")
    h.forward(db2, out, hstu.HSTU_MASK_MFALCON)
    assert h.device_error() == 0
    h.close()


def test_deterministic_and_stack_equals_layer_sequence():
    w = wl.WORKLOADS[1]
    batch = wl.make_batch(w, num_users=12)
    batch.layers = batch.layers + wl.make_custom_batch([4], w.d_model, w.num_heads, seed=5,
                                                       num_layers=2).layers
    cfg = runtime.config_for(w, batch.total_tokens, batch.num_users)
    h = runtime.Handle(cfg, 0)
    db = runtime.to_device(batch, w.storage, w.compute, "cuda:0")
    a = torch.empty_like(db.x)
    b = torch.empty_like(db.x)
    h.forward(db, a, hstu.HSTU_MASK_CAUSAL)             # 3-layer stack
    h.forward(db, b, hstu.HSTU_MASK_CAUSAL)
    assert torch.equal(a, b)
    c = db.x.clone()
    for l in range(3):
        nxt = torch.empty_like(c)
        h.forward(db, nxt, hstu.HSTU_MASK_CAUSAL, layers=[db.layers[l]], x=c)
        c = nxt
    assert torch.equal(a, c)
    # in place: out aliases values
    d = db.x.clone()
    h.forward(db, d, hstu.HSTU_MASK_CAUSAL, x=d)
    assert torch.equal(a, d)
    assert h.device_error() == 0
    h.close()


def test_packing_and_prefix_invariance_on_gpu():
    """Per-user rows do not depend on packing order; causal prefixes do not see the future."""
    d, H = 256, 4
    lengths = [200, 0, 77, 301, 5]
    batch = wl.make_custom_batch(lengths, d, H, seed=99, weight_scale=0.05, rab_scale=0.5)
    base = gpu_run(batch, "bf16", "bf16", d=d, H=H, n_norm=512, mask="causal", want=("AV",))
    offs = batch.seq_offsets
    order = [3, 1, 4, 0, 2]
    rows = np.concatenate([np.arange(offs[b], offs[b + 1]) for b in order])
    perm = wl.Batch(lengths=batch.lengths[order], seq_offsets=wl.offsets_from_lengths(batch.lengths[order]),
                    timestamps=batch.timestamps[rows], num_candidates=batch.num_candidates[order],
                    x=batch.x[rows], layers=batch.layers)
    pr = gpu_run(perm, "bf16", "bf16", d=d, H=H, n_norm=512, mask="causal", want=("AV",))
    assert rel_err(pr["AV"], base["AV"][rows]) <= 1e-5
    assert np.max(np.abs(pr["Y"] - base["Y"][rows])) <= 2.0 ** -7 * np.max(np.abs(base["Y"]))
    # prefix: keep the first 100 tokens of every user
    keep = np.concatenate([np.arange(offs[b], offs[b] + min(100, lengths[b])) for b in range(5)])
    lp = np.minimum(batch.lengths, 100)
    pre = wl.Batch(lengths=lp, seq_offsets=wl.offsets_from_lengths(lp),
                   timestamps=batch.timestamps[keep], num_candidates=batch.num_candidates,
                   x=batch.x[keep], layers=batch.layers)
    pp = gpu_run(pre, "bf16", "bf16", d=d, H=H, n_norm=512, mask="causal", want=("AV",))
    assert rel_err(pp["AV"], base["AV"][keep]) <= 1e-5
