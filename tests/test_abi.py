"""The C-ABI library loads and exports every declared entry point; host-side
logic (argument checks, the time-bucket threshold table) runs without a GPU."""
import ctypes
import os

import numpy as np
import pytest

import oracle
from jagged_pointwise_attention_hstu_b200 import build, hstu


@pytest.fixture(scope="module")
def lib():
    build.build()
    return hstu.load()


def test_every_declared_symbol_is_exported(lib):
    names = hstu.declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(7):
        assert hstu.status_string(s).startswith("HSTU_")
    assert hstu.status_string(99) == "HSTU_ERR_UNKNOWN"


@pytest.mark.parametrize("div,nb", [(0.301, 128), (0.5, 64), (0.1, 256)])
def test_time_thresholds_reproduce_the_bucket_rule(lib, div, nb):
    """The library's integer thresholds give exactly the oracle's fp64 buckets."""
    thr = np.array(hstu.hstu_time_bucket_thresholds(div, nb), dtype=np.int64)
    assert thr[0] == 0 and np.all(np.diff(thr) >= 0)
    reach = thr < 2 ** 62
    k = np.nonzero(reach)[0][1:]
    # at each threshold the bucket reaches k; one second earlier it is below k
    assert np.all(oracle.time_bucket(thr[k], div, nb) >= k)
    assert np.all(oracle.time_bucket(thr[k] - 1, div, nb) < k)
    # bucket(dt) = #{k >= 1 : dt >= thr[k]} on a dense and a wide sample of gaps
    rng = np.random.default_rng(0)
    dts = np.concatenate([np.arange(0, 5000), rng.integers(0, 2 ** 40, 20000),
                          np.unique(thr[reach]) + 1, np.unique(thr[reach]) - 1])
    dts = dts[dts >= 0]
    mine = (dts[:, None] >= thr[None, 1:]).sum(axis=1)
    assert np.array_equal(mine, oracle.time_bucket(dts, div, nb))


def _cfg(**kw):
    base = dict(io_dtype=hstu.HSTU_DTYPE_BF16, compute_dtype=hstu.HSTU_DTYPE_BF16, n_norm=0,
                pos_buckets=129, pos_clamp=128, time_buckets=128, time_log_div=0.301,
                ln_eps=1e-5, max_tokens=1024, max_users=8)
    d = kw.pop("d", 256)
    H = kw.pop("H", 4)
    base.update(kw)
    return hstu.make_config(d, H, **base)


@pytest.mark.parametrize("kw,status", [
    (dict(d=256, H=3), hstu.HSTU_ERR_INVALID_ARG),          # d != H * hd
    (dict(d=256, H=8), hstu.HSTU_ERR_UNSUPPORTED),          # hd 32 on the tensor-core path
    (dict(pos_clamp=129), hstu.HSTU_ERR_INVALID_ARG),       # clamp outside the table
    (dict(time_buckets=0), hstu.HSTU_ERR_INVALID_ARG),
    (dict(time_log_div=0.0), hstu.HSTU_ERR_INVALID_ARG),
    (dict(max_tokens=2 ** 31), hstu.HSTU_ERR_INVALID_ARG),
    (dict(max_tokens=2 ** 30 + 1), hstu.HSTU_ERR_INVALID_ARG),  # 32-bit row indices
    (dict(max_tokens=-1), hstu.HSTU_ERR_INVALID_ARG),
    (dict(io_dtype=7), hstu.HSTU_ERR_INVALID_ARG),
    (dict(compute_dtype=hstu.HSTU_DTYPE_FP32), hstu.HSTU_ERR_UNSUPPORTED),  # fp32 math, bf16 io
    (dict(d=320, H=5), hstu.HSTU_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_configs_before_touching_cuda(lib, kw, status):
    h = ctypes.c_void_p()
    cfg = _cfg(**kw)
    assert lib.hstu_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == status
    assert not h.value


def test_null_arguments_are_rejected(lib):
    assert lib.hstu_create(None, 0, None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_destroy(None) == hstu.HSTU_OK
    w = hstu.hstu_layer_weights()
    assert lib.hstu_layer_forward(None, None, 0, None, 0, None, ctypes.byref(w), 0, None, None,
                                  None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_get_device_error(None, None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_time_bucket_thresholds(0.301, 0, None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_debug_umma_tile(0, None, None, None, 128, 64) == hstu.HSTU_ERR_INVALID_ARG
    c = ctypes.c_void_p()
    assert lib.hstu_cache_create(None, 1, 16, 256, ctypes.byref(c)) == hstu.HSTU_ERR_INVALID_ARG
    assert not c.value
    assert lib.hstu_cache_create(None, 1, 16, 256, None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_cache_destroy(None) == hstu.HSTU_OK
    assert lib.hstu_cache_prefill(None, None, None, 0, None, 0, None, ctypes.byref(w), 1, None,
                                  None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_cache_score(None, None, None, None, None, ctypes.byref(w), 1, None,
                                None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_attention_backward(None, None, None, 0, None, 0, None, 0, None, None, None,
                                       None, None, None, None, None,
                                       None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_attention_forward(None, None, 0, None, 0, None, 0, None, None, None, None,
                                      None) == hstu.HSTU_ERR_INVALID_ARG
    assert lib.hstu_set_wait_limit(None, 0) == hstu.HSTU_ERR_INVALID_ARG


def test_stochastic_length_host_checks(lib):
    """Scratch sizing and argument checks return before touching CUDA."""
    assert lib.hstu_stochastic_length_scratch_bytes(0, 0) == 256
    assert lib.hstu_stochastic_length_scratch_bytes(1000, 10) == 256 + 256 + 1024
    assert lib.hstu_stochastic_length_scratch_bytes(-1, 1) == 0
    P = 256    # a non-null, 256-aligned stand-in pointer; never dereferenced here
    bad = [
        dict(B=-1), dict(T=-1), dict(T=2 ** 31), dict(B=0, T=5), dict(n_c=0),
        dict(alpha=float("nan")), dict(alpha=float("inf")), dict(offsets=None),
        dict(out_offsets=None), dict(scratch=None), dict(scratch=P + 16), dict(u=None),
        dict(keys=None), dict(out_index=None), dict(ts=P, out_ts=None),
        dict(values=P, out_values=None), dict(values=P, out_values=P, row_bytes=24),
        dict(values=P, out_values=P, row_bytes=0), dict(values=P + 8, out_values=P),
    ]
    for over in bad:
        a = dict(offsets=P, B=2, T=100, u=P, keys=P, n_c=776, alpha=1.6, values=None,
                 row_bytes=0, ts=None, out_offsets=P, out_index=P, out_values=None,
                 out_ts=None, scratch=P, err=None)
        a.update(over)
        st = lib.hstu_stochastic_length(a["offsets"], a["B"], a["T"], a["u"], a["keys"], a["n_c"],
                                        a["alpha"], a["values"], a["row_bytes"], a["ts"],
                                        a["out_offsets"], a["out_index"], a["out_values"],
                                        a["out_ts"], a["scratch"], a["err"], None)
        assert st == hstu.HSTU_ERR_INVALID_ARG, over


def test_plain_c_consumer_compiles_links_and_runs(tmp_path):
    """include/hstu.h is plain C99; a C program links every entry point of
    libhstu.so and calls the host-only ones."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(hstu.LIB_PATH)
    exe = str(tmp_path / "abi_consumer")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c", "abi_consumer.c"), "-o", exe,
                    "-L", libdir, "-lhstu", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    declared = hstu.declared_symbols()
    assert out[0] == f"entry_points {len(declared)}"
    thr = hstu.hstu_time_bucket_thresholds(0.301, 128)
    assert out[1] == f"thresholds {thr[0]} {thr[1]} {thr[3]} {thr[40]}"
    assert out[2] == "status HSTU_ERR_WORKSPACE"
    assert out[3] == f"create {hstu.HSTU_ERR_INVALID_ARG} null"
    assert out[4] == "sl_scratch 1536"
