"""ctypes binding of libhstu.so: the C-ABI entry points under the same names.

Argument marshalling only: every step of the layer forward runs in the CUDA
library.  Tensors are passed as raw device pointers (``tensor.data_ptr()``);
PyTorch is used by callers for device memory and streams.  If the library is
missing, every call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import (POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_int64, c_size_t,
                    c_uint8, c_void_p)
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhstu.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "hstu.h")

HSTU_OK = 0
HSTU_ERR_INVALID_ARG = 1
HSTU_ERR_UNSUPPORTED = 2
HSTU_ERR_WORKSPACE = 3
HSTU_ERR_CUDA = 4
HSTU_ERR_DEVICE_CHECK = 5
HSTU_ERR_TIMEOUT = 6

HSTU_DTYPE_BF16 = 0
HSTU_DTYPE_FP32 = 1
HSTU_MASK_CAUSAL = 0
HSTU_MASK_MFALCON = 1

HSTU_DEVERR_OFFSETS = 0x1
HSTU_DEVERR_CANDIDATES = 0x2
HSTU_DEVERR_TIMESTAMPS = 0x4
HSTU_DEVERR_TIMEOUT = 0x8

HSTU_TENSOR_UVQK = 0
HSTU_TENSOR_AV = 1
HSTU_TENSOR_G = 2


class HstuError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class hstu_layer_grads(ctypes.Structure):
    _fields_ = [("w1", c_void_p), ("b1", c_void_p), ("w2", c_void_p), ("b2", c_void_p),
                ("ln_gamma", c_void_p), ("ln_beta", c_void_p), ("rab_pos", c_void_p),
                ("rab_time", c_void_p)]


class hstu_config(ctypes.Structure):
    _fields_ = [("d_model", c_int32), ("num_heads", c_int32), ("head_dim", c_int32),
                ("io_dtype", c_int), ("compute_dtype", c_int), ("n_norm", c_int32),
                ("pos_buckets", c_int32), ("pos_clamp", c_int32), ("time_buckets", c_int32),
                ("time_log_div", c_double), ("ln_eps", c_float), ("max_tokens", c_int64),
                ("max_users", c_int32)]


class hstu_layer_weights(ctypes.Structure):
    _fields_ = [("w1", c_void_p), ("b1", c_void_p), ("w2", c_void_p), ("b2", c_void_p),
                ("ln_gamma", c_void_p), ("ln_beta", c_void_p), ("rab_pos", c_void_p),
                ("rab_time", c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    """Loads libhstu.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m jagged_pointwise_attention_hstu_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    H = c_void_p
    sig = {
        "hstu_create": (c_int, [POINTER(hstu_config), c_int32, POINTER(H)]),
        "hstu_destroy": (c_int, [H]),
        "hstu_layer_forward": (c_int, [H, c_void_p, c_int64, c_void_p, c_int32, c_void_p,
                                       POINTER(hstu_layer_weights), c_int, c_void_p, c_void_p,
                                       c_void_p]),
        "hstu_stack_forward": (c_int, [H, c_void_p, c_int64, c_void_p, c_int32, c_void_p,
                                       POINTER(hstu_layer_weights), c_int32, c_int, c_void_p,
                                       c_void_p, c_void_p]),
        "hstu_status_string": (c_char_p, [c_int]),
        "hstu_get_device_error": (c_int, [H, POINTER(c_int32)]),
        "hstu_time_bucket_thresholds": (c_int, [c_double, c_int32, POINTER(c_int64)]),
        "hstu_copy_intermediate": (c_int, [H, c_int, c_void_p, c_size_t, c_void_p]),
        "hstu_debug_attention_buckets": (c_int, [H, c_int64, c_void_p, c_int32, c_void_p, c_int,
                                                 c_void_p, c_void_p, c_void_p, c_void_p]),
        "hstu_debug_umma_tile": (c_int, [c_int32, c_void_p, c_void_p, c_void_p, c_int32,
                                         c_int32]),
        "hstu_attention_noalloc": (c_int, [POINTER(hstu_config), c_void_p, c_int64, c_void_p,
                                           c_int32, c_void_p, c_int, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p]),
        "hstu_cache_create": (c_int, [H, c_int32, c_int64, c_int64, POINTER(c_void_p)]),
        "hstu_cache_destroy": (c_int, [c_void_p]),
        "hstu_cache_prefill": (c_int, [H, c_void_p, c_void_p, c_int64, c_void_p, c_int32,
                                       c_void_p, POINTER(hstu_layer_weights), c_int32, c_void_p,
                                       c_void_p]),
        "hstu_cache_score": (c_int, [H, c_void_p, c_void_p, POINTER(c_int32), c_void_p,
                                     POINTER(hstu_layer_weights), c_int32, c_void_p, c_void_p]),
        "hstu_stochastic_length_scratch_bytes": (c_size_t, [c_int64, c_int32]),
        "hstu_stochastic_length": (c_int, [c_void_p, c_int32, c_int64, c_void_p, c_void_p,
                                           c_int32, c_double, c_void_p, c_int64, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p]),
        "hstu_attention_forward": (c_int, [H, c_void_p, c_int64, c_void_p, c_int32, c_void_p,
                                           c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p]),
        "hstu_attention_backward": (c_int, [H, c_void_p, c_void_p, c_int64, c_void_p, c_int32,
                                            c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_void_p]),
        "hstu_layer_backward": (c_int, [H, c_void_p, c_void_p, c_void_p, c_void_p, c_int64,
                                        c_void_p, c_int32, c_void_p,
                                        POINTER(hstu_layer_weights), c_int, c_void_p, c_void_p,
                                        POINTER(hstu_layer_grads), c_void_p]),
        "hstu_set_wait_limit": (c_int, [H, c_int64]),
        "hstu_set_kernel_timing": (c_int, [H, c_int32]),
        "hstu_get_kernel_timing": (c_int, [H, POINTER(c_double), POINTER(c_int64)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def declared_symbols() -> list:
    """Names of the functions declared in include/hstu.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(hstu_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return load().hstu_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != HSTU_OK:
        raise HstuError(status, what)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------- entry points

def hstu_create(cfg: hstu_config, device: int = 0) -> c_void_p:
    h = c_void_p()
    _check(load().hstu_create(ctypes.byref(cfg), device, ctypes.byref(h)), "hstu_create")
    return h


def hstu_destroy(handle) -> None:
    _check(load().hstu_destroy(handle), "hstu_destroy")


def hstu_layer_weights_of(w1, b1, w2, b2, ln_gamma, ln_beta, rab_pos, rab_time) -> hstu_layer_weights:
    return hstu_layer_weights(_ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(ln_gamma),
                              _ptr(ln_beta), _ptr(rab_pos), _ptr(rab_time))


def hstu_layer_forward(handle, values, total_tokens: int, seq_offsets, num_users: int, timestamps,
                       weights: hstu_layer_weights, mask_mode: int, num_candidates, out,
                       stream=None) -> None:
    _check(load().hstu_layer_forward(handle, _ptr(values), total_tokens, _ptr(seq_offsets),
                                     num_users, _ptr(timestamps), ctypes.byref(weights), mask_mode,
                                     _ptr(num_candidates), _ptr(out), _stream_ptr(stream)),
           "hstu_layer_forward")


def hstu_stack_forward(handle, values, total_tokens: int, seq_offsets, num_users: int, timestamps,
                       layers: Sequence[hstu_layer_weights], mask_mode: int, num_candidates, out,
                       stream=None) -> None:
    arr = (hstu_layer_weights * len(layers))(*layers)
    _check(load().hstu_stack_forward(handle, _ptr(values), total_tokens, _ptr(seq_offsets),
                                     num_users, _ptr(timestamps), arr, len(layers), mask_mode,
                                     _ptr(num_candidates), _ptr(out), _stream_ptr(stream)),
           "hstu_stack_forward")


def hstu_get_device_error(handle) -> int:
    """Returns the device error bits (0 = none) and clears them."""
    bits = c_int32(0)
    st = load().hstu_get_device_error(handle, ctypes.byref(bits))
    if st not in (HSTU_OK, HSTU_ERR_DEVICE_CHECK, HSTU_ERR_TIMEOUT):
        _check(st, "hstu_get_device_error")
    return int(bits.value)


def hstu_time_bucket_thresholds(time_log_div: float, num_buckets: int) -> list:
    out = (c_int64 * num_buckets)()
    _check(load().hstu_time_bucket_thresholds(time_log_div, num_buckets, out),
           "hstu_time_bucket_thresholds")
    return list(out)


def hstu_copy_intermediate(handle, which: int, dst, nbytes: int, stream=None) -> None:
    _check(load().hstu_copy_intermediate(handle, which, _ptr(dst), nbytes, _stream_ptr(stream)),
           "hstu_copy_intermediate")


def hstu_debug_attention_buckets(handle, total_tokens: int, seq_offsets, num_users: int,
                                 timestamps, mask_mode: int, num_candidates, pidx_out, tidx_out,
                                 vis_out) -> None:
    _check(load().hstu_debug_attention_buckets(handle, total_tokens, _ptr(seq_offsets), num_users,
                                               _ptr(timestamps), mask_mode, _ptr(num_candidates),
                                               _ptr(pidx_out), _ptr(tidx_out), _ptr(vis_out)),
           "hstu_debug_attention_buckets")


def hstu_debug_umma_tile(mode: int, a, b, c, n: int, k: int) -> None:
    _check(load().hstu_debug_umma_tile(mode, _ptr(a), _ptr(b), _ptr(c), n, k),
           "hstu_debug_umma_tile")


HSTU_NOALLOC_MAX_TOKENS = 65536


def hstu_attention_noalloc(cfg: hstu_config, uvqk, total_tokens: int, seq_offsets, num_users: int,
                           timestamps, mask_mode: int, num_candidates, rab_pos, rab_time, av,
                           device_error=None, stream=None) -> None:
    _check(load().hstu_attention_noalloc(ctypes.byref(cfg), _ptr(uvqk), total_tokens,
                                         _ptr(seq_offsets), num_users, _ptr(timestamps), mask_mode,
                                         _ptr(num_candidates), _ptr(rab_pos), _ptr(rab_time),
                                         _ptr(av), _ptr(device_error), _stream_ptr(stream)),
           "hstu_attention_noalloc")


def hstu_cache_create(handle, num_layers: int, max_history_tokens: int,
                      max_candidate_rows: int) -> c_void_p:
    c = c_void_p()
    _check(load().hstu_cache_create(handle, num_layers, max_history_tokens, max_candidate_rows,
                                    ctypes.byref(c)), "hstu_cache_create")
    return c


def hstu_cache_destroy(cache) -> None:
    _check(load().hstu_cache_destroy(cache), "hstu_cache_destroy")


def hstu_cache_prefill(handle, cache, values, total_tokens: int, seq_offsets, num_users: int,
                       timestamps, layers: Sequence[hstu_layer_weights], out, stream=None) -> None:
    arr = (hstu_layer_weights * len(layers))(*layers)
    _check(load().hstu_cache_prefill(handle, cache, _ptr(values), total_tokens, _ptr(seq_offsets),
                                     num_users, _ptr(timestamps), arr, len(layers), _ptr(out),
                                     _stream_ptr(stream)),
           "hstu_cache_prefill")


def hstu_cache_score(handle, cache, values, num_candidates: Sequence[int], timestamps,
                     layers: Sequence[hstu_layer_weights], out, stream=None) -> None:
    """num_candidates: host integers, one per user of the prefill."""
    counts = (c_int32 * max(len(num_candidates), 1))(*[int(n) for n in num_candidates])
    arr = (hstu_layer_weights * len(layers))(*layers)
    _check(load().hstu_cache_score(handle, cache, _ptr(values), counts, _ptr(timestamps), arr,
                                   len(layers), _ptr(out), _stream_ptr(stream)),
           "hstu_cache_score")


HSTU_SL_MAX_SAMPLED_LEN = 8192
HSTU_DEVERR_SL_TOO_LONG = 0x10


def hstu_stochastic_length_scratch_bytes(total_tokens: int, num_users: int) -> int:
    return int(load().hstu_stochastic_length_scratch_bytes(total_tokens, num_users))


def hstu_stochastic_length(seq_offsets, num_users: int, total_tokens: int, user_uniform,
                           token_keys, n_c: int, alpha: float, values, row_bytes: int,
                           timestamps, out_offsets, out_index, out_values, out_timestamps,
                           scratch, device_error=None, stream=None) -> None:
    _check(load().hstu_stochastic_length(_ptr(seq_offsets), num_users, total_tokens,
                                         _ptr(user_uniform), _ptr(token_keys), n_c, alpha,
                                         _ptr(values), row_bytes, _ptr(timestamps),
                                         _ptr(out_offsets), _ptr(out_index), _ptr(out_values),
                                         _ptr(out_timestamps), _ptr(scratch),
                                         _ptr(device_error), _stream_ptr(stream)),
           "hstu_stochastic_length")


def hstu_attention_forward(handle, uvqk, total_tokens: int, seq_offsets, num_users: int,
                           timestamps, mask_mode: int, num_candidates, rab_pos, rab_time, av,
                           stream=None) -> None:
    _check(load().hstu_attention_forward(handle, _ptr(uvqk), total_tokens, _ptr(seq_offsets),
                                         num_users, _ptr(timestamps), mask_mode,
                                         _ptr(num_candidates), _ptr(rab_pos), _ptr(rab_time),
                                         _ptr(av), _stream_ptr(stream)),
           "hstu_attention_forward")


def hstu_attention_backward(handle, uvqk, d_out, total_tokens: int, seq_offsets, num_users: int,
                            timestamps, mask_mode: int, num_candidates, rab_pos, rab_time, dq, dk,
                            dv, d_rab_pos, d_rab_time, stream=None) -> None:
    _check(load().hstu_attention_backward(handle, _ptr(uvqk), _ptr(d_out), total_tokens,
                                          _ptr(seq_offsets), num_users, _ptr(timestamps),
                                          mask_mode, _ptr(num_candidates), _ptr(rab_pos),
                                          _ptr(rab_time), _ptr(dq), _ptr(dk), _ptr(dv),
                                          _ptr(d_rab_pos), _ptr(d_rab_time), _stream_ptr(stream)),
           "hstu_attention_backward")


def hstu_layer_backward(handle, values, uvqk, av, d_out, total_tokens: int, seq_offsets,
                        num_users: int, timestamps, weights: hstu_layer_weights, mask_mode: int,
                        num_candidates, d_values, grads: dict, stream=None) -> None:
    """grads: dict of fp32 device tensors w1, b1, w2, b2, ln_gamma, ln_beta, rab_pos, rab_time."""
    g = hstu_layer_grads(*[_ptr(grads[k]) for k in ("w1", "b1", "w2", "b2", "ln_gamma",
                                                    "ln_beta", "rab_pos", "rab_time")])
    _check(load().hstu_layer_backward(handle, _ptr(values), _ptr(uvqk), _ptr(av), _ptr(d_out),
                                      total_tokens, _ptr(seq_offsets), num_users,
                                      _ptr(timestamps), ctypes.byref(weights), mask_mode,
                                      _ptr(num_candidates), _ptr(d_values), ctypes.byref(g),
                                      _stream_ptr(stream)),
           "hstu_layer_backward")


def hstu_set_wait_limit(handle, cycles: int) -> None:
    _check(load().hstu_set_wait_limit(handle, cycles), "hstu_set_wait_limit")


KERNEL_KINDS = ("schedule", "cast", "f1", "attention", "ln_gate", "f2", "block")


def hstu_set_kernel_timing(handle, enabled: bool) -> None:
    _check(load().hstu_set_kernel_timing(handle, 1 if enabled else 0), "hstu_set_kernel_timing")


def hstu_get_kernel_timing(handle) -> dict:
    """{kind: (total_ms, launches)} for every kernel kind."""
    ms = (c_double * len(KERNEL_KINDS))()
    n = (c_int64 * len(KERNEL_KINDS))()
    _check(load().hstu_get_kernel_timing(handle, ms, n), "hstu_get_kernel_timing")
    return {k: (ms[i], n[i]) for i, k in enumerate(KERNEL_KINDS)}


def make_config(d_model: int, num_heads: int, *, io_dtype: int, compute_dtype: int, n_norm: int,
                pos_buckets: int, pos_clamp: int, time_buckets: int, time_log_div: float,
                ln_eps: float, max_tokens: int, max_users: int) -> hstu_config:
    return hstu_config(d_model, num_heads, d_model // num_heads, io_dtype, compute_dtype, n_norm,
                       pos_buckets, pos_clamp, time_buckets, time_log_div, ln_eps, max_tokens,
                       max_users)
