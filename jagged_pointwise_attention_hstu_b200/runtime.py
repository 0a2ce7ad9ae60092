"""Device-side plumbing above the C ABI: tensors in HBM, handles, streams.

Moves a seeded batch into device memory in the dtypes the library expects and
wraps a handle; the forward itself is one C-ABI call.  Nothing here computes
any part of the layer.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import hstu
from .workloads import Batch, Workload

_TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32}


@dataclass
class DeviceLayer:
    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor
    ln_gamma: torch.Tensor
    ln_beta: torch.Tensor
    rab_pos: torch.Tensor
    rab_time: torch.Tensor

    def struct(self) -> hstu.hstu_layer_weights:
        return hstu.hstu_layer_weights_of(self.w1, self.b1, self.w2, self.b2, self.ln_gamma,
                                          self.ln_beta, self.rab_pos, self.rab_time)


@dataclass
class DeviceBatch:
    x: torch.Tensor               # [T, d] storage dtype
    seq_offsets: torch.Tensor     # int32 [B+1]
    timestamps: torch.Tensor      # int64 [T]
    num_candidates: torch.Tensor  # int32 [B]
    layers: List[DeviceLayer]
    total_tokens: int
    num_users: int


def device_layers(batch: Batch, compute: str, device) -> List[DeviceLayer]:
    wdt = _TORCH_DTYPE[compute]
    f32 = dict(dtype=torch.float32, device=device)
    out = []
    for lp in batch.layers:
        out.append(DeviceLayer(
            w1=torch.from_numpy(lp.w1).to(device=device, dtype=wdt).contiguous(),
            b1=torch.from_numpy(lp.b1).to(**f32).contiguous(),
            w2=torch.from_numpy(lp.w2).to(device=device, dtype=wdt).contiguous(),
            b2=torch.from_numpy(lp.b2).to(**f32).contiguous(),
            ln_gamma=torch.from_numpy(lp.ln_gamma).to(**f32).contiguous(),
            ln_beta=torch.from_numpy(lp.ln_beta).to(**f32).contiguous(),
            rab_pos=torch.from_numpy(lp.rab_pos).to(**f32).contiguous(),
            rab_time=torch.from_numpy(lp.rab_time).to(**f32).contiguous()))
    return out


def to_device(batch: Batch, storage: str, compute: str, device="cuda") -> DeviceBatch:
    x = torch.from_numpy(batch.x).to(device=device, dtype=_TORCH_DTYPE[storage]).contiguous()
    if x.numel() == 0:
        x = torch.empty((0, batch.x.shape[1]), dtype=_TORCH_DTYPE[storage], device=device)
    return DeviceBatch(
        x=x,
        seq_offsets=torch.from_numpy(batch.seq_offsets.astype(np.int32)).to(device),
        timestamps=torch.from_numpy(batch.timestamps.astype(np.int64)).to(device),
        num_candidates=torch.from_numpy(batch.num_candidates.astype(np.int32)).to(device),
        layers=device_layers(batch, compute, device),
        total_tokens=batch.total_tokens, num_users=batch.num_users)


def config_for(w: Workload, max_tokens: int, max_users: int) -> hstu.hstu_config:
    return hstu.make_config(
        w.d_model, w.num_heads,
        io_dtype=hstu.HSTU_DTYPE_BF16 if w.storage == "bf16" else hstu.HSTU_DTYPE_FP32,
        compute_dtype=hstu.HSTU_DTYPE_BF16 if w.compute == "bf16" else hstu.HSTU_DTYPE_FP32,
        n_norm=w.n_norm, pos_buckets=w.pos_buckets, pos_clamp=w.pos_clamp,
        time_buckets=w.time_buckets, time_log_div=w.time_log_div, ln_eps=w.ln_eps,
        max_tokens=max_tokens, max_users=max_users)


class Handle:
    """Owns one C-ABI handle (workspace on one GPU)."""

    def __init__(self, cfg: hstu.hstu_config, device: int = 0):
        self.cfg = cfg
        self.device = device
        self.h = hstu.hstu_create(cfg, device)

    def close(self):
        if self.h is not None:
            hstu.hstu_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, db: DeviceBatch, out: torch.Tensor, mask_mode: int,
                layers: Optional[List[DeviceLayer]] = None, x: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        """Runs every layer of ``layers`` (default: the batch's) as one stack call."""
        layers = db.layers if layers is None else layers
        xin = db.x if x is None else x
        if stream is None:
            stream = torch.cuda.current_stream(out.device)
        structs = [l.struct() for l in layers]
        if len(structs) == 1:
            hstu.hstu_layer_forward(self.h, xin, db.total_tokens, db.seq_offsets, db.num_users,
                                    db.timestamps, structs[0], mask_mode, db.num_candidates, out,
                                    stream)
        else:
            hstu.hstu_stack_forward(self.h, xin, db.total_tokens, db.seq_offsets, db.num_users,
                                    db.timestamps, structs, mask_mode, db.num_candidates, out,
                                    stream)
        return out

    def train_step(self, db: DeviceBatch, mask_mode: int, dy: torch.Tensor, saved: dict,
                   grads: List[dict], stream=None) -> torch.Tensor:
        """One forward and backward pass of the stack through the C ABI.

        The forward runs layer by layer and keeps each layer's input and the
        U|V|Q|K and O the backward reads (``saved``: preallocated lists "x",
        "uvqk", "av" of per-layer device tensors, "y" and "dx" [T, d]); the
        backward walks the
        layers in reverse with hstu_layer_backward, filling ``grads[l]`` and
        returning dX of the stack's input."""
        if stream is None:
            stream = torch.cuda.current_stream(dy.device)
        T = db.total_tokens
        L = len(db.layers)
        saved["x"][0].copy_(db.x)
        for l in range(L):
            out = saved["x"][l + 1] if l + 1 < L else saved["y"]
            hstu.hstu_layer_forward(self.h, saved["x"][l], T, db.seq_offsets, db.num_users,
                                    db.timestamps, db.layers[l].struct(), mask_mode,
                                    db.num_candidates, out, stream)
            u, a = saved["uvqk"][l], saved["av"][l]
            hstu.hstu_copy_intermediate(self.h, hstu.HSTU_TENSOR_UVQK, u,
                                        u.numel() * u.element_size(), stream)
            hstu.hstu_copy_intermediate(self.h, hstu.HSTU_TENSOR_AV, a,
                                        a.numel() * a.element_size(), stream)
        g = dy
        for l in reversed(range(L)):
            dx = saved["dx"]
            hstu.hstu_layer_backward(self.h, saved["x"][l], saved["uvqk"][l], saved["av"][l], g,
                                     T, db.seq_offsets, db.num_users, db.timestamps,
                                     db.layers[l].struct(), mask_mode, db.num_candidates, dx,
                                     grads[l], stream)
            g = dx
        return g

    def intermediate(self, which: int, T: int) -> torch.Tensor:
        d = self.cfg.d_model
        cdt = torch.bfloat16 if self.cfg.compute_dtype == hstu.HSTU_DTYPE_BF16 else torch.float32
        if which == hstu.HSTU_TENSOR_UVQK:
            t = torch.empty((T, 4 * d), dtype=cdt, device=f"cuda:{self.device}")
        elif which == hstu.HSTU_TENSOR_AV:
            t = torch.empty((T, d), dtype=torch.float32, device=f"cuda:{self.device}")
        else:
            t = torch.empty((T, d), dtype=cdt, device=f"cuda:{self.device}")
        hstu.hstu_copy_intermediate(self.h, which, t, t.numel() * t.element_size(),
                                    torch.cuda.current_stream(t.device))
        return t

    def device_error(self) -> int:
        return hstu.hstu_get_device_error(self.h)


def mask_mode_of(w: Workload) -> int:
    return hstu.HSTU_MASK_MFALCON if w.mask == "mfalcon" else hstu.HSTU_MASK_CAUSAL
