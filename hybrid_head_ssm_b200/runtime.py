"""Device-memory plumbing around the C ABI: uploads a layer's weights, allocates the
KV buffers, SSM state and workspace as torch CUDA tensors, and calls
hymba_mixer_prefill / hymba_mixer_decode on torch's current stream. No arithmetic
of the mixer happens here.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional

import numpy as np
import torch

from . import (HYMBA_BF16, HYMBA_MODE_DECODE, HYMBA_MODE_PREFILL, check, cfg_struct,
               current_stream_ptr, hymba_mixer_decode, hymba_mixer_prefill, hymba_workspace_bytes,
               kv_struct, state_struct, weights_struct)

BIG = ("w_in", "w_dt", "w_out", "meta")
NAMES = ("w_in", "w_dt", "b_dt", "conv_w", "conv_b", "A_log", "D", "norm_attn_w", "norm_ssm_w",
         "beta1", "beta2", "w_out", "meta", "kv_scale", "kv_bias", "pre_norm_w")
# a consumer's affine adaptation of the shared K/V; the block's pre-mixer norm gain
OPTIONAL = ("kv_scale", "kv_bias", "pre_norm_w")


def act_dtype(cfg):
    return torch.bfloat16 if cfg.dtype == HYMBA_BF16 else torch.float32


def mid_dtype(cfg):
    """Element type of K/V and the other intermediates (fp16 in bf16 layers)."""
    return torch.float16 if cfg.dtype == HYMBA_BF16 else torch.float32


class DeviceLayer:
    """One mixer layer's weights in device memory and its C structs."""

    def __init__(self, cfg, w: Dict[str, np.ndarray], device="cuda"):
        self.cfg = cfg
        self.c = cfg_struct(cfg)
        adt = act_dtype(cfg)
        self.t = {}
        for n in NAMES:
            a = w.get(n)
            if a is None and n in OPTIONAL:
                continue
            a = w[n]
            dt = adt if n in BIG else torch.float32
            self.t[n] = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=dt)
        self.s = weights_struct(self.t)


class KV:
    """K/V buffers of a producer layer (and its consumers)."""

    def __init__(self, cfg, B: int, seq_cap: int = 0, cache_cap: int = 0, device="cuda"):
        adt = mid_dtype(cfg)
        G, dh, dv = cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
        self.k_seq = torch.empty((B, G, seq_cap, dh), dtype=adt, device=device) if seq_cap else None
        self.v_seq = torch.empty((B, G, seq_cap, dv), dtype=adt, device=device) if seq_cap else None
        self.k_cache = torch.zeros((B, G, cache_cap, dh), dtype=adt, device=device) if cache_cap else None
        self.v_cache = torch.zeros((B, G, cache_cap, dv), dtype=adt, device=device) if cache_cap else None
        self.len = torch.zeros(B, dtype=torch.int32, device=device) if cache_cap else None
        self.s = kv_struct(cfg, B, self.k_seq, self.v_seq, self.k_cache, self.v_cache, self.len)


class State:
    def __init__(self, cfg, B: int, device="cuda"):
        self.h = torch.zeros((B, cfg.d_inner, cfg.d_state), dtype=torch.float32, device=device)
        self.conv = torch.zeros((B, cfg.d_inner, cfg.d_conv), dtype=torch.float32, device=device)
        self.s = state_struct(self.h, self.conv)


def workspace(cfg, B: int, T: int, mode: int, device="cuda") -> torch.Tensor:
    n = hymba_workspace_bytes(ctypes.byref(cfg_struct(cfg)), B, T, mode)
    if n == 0:
        raise ValueError("invalid layer configuration")
    return torch.empty(n, dtype=torch.uint8, device=device)


def prefill(layer: DeviceLayer, x: torch.Tensor, T: int, kv: KV, y: torch.Tensor, ws: torch.Tensor,
            state: Optional[State] = None, flags: int = 0, kv_struct_override=None) -> None:
    kvs = kv_struct_override if kv_struct_override is not None else kv.s
    check(hymba_mixer_prefill(ctypes.byref(layer.c), ctypes.byref(layer.s), x.data_ptr(), x.shape[0], T,
                              flags, y.data_ptr(), ctypes.byref(kvs),
                              ctypes.byref(state.s) if state is not None else None,
                              ws.data_ptr(), ws.numel(), current_stream_ptr()))


def decode(layer: DeviceLayer, x_t: torch.Tensor, kv_s, state: State, y_t: torch.Tensor,
           ws: torch.Tensor, flags: int = 0) -> None:
    check(hymba_mixer_decode(ctypes.byref(layer.c), ctypes.byref(layer.s), x_t.data_ptr(), x_t.shape[0],
                             flags, y_t.data_ptr(), ctypes.byref(kv_s), ctypes.byref(state.s),
                             ws.data_ptr(), ws.numel(), current_stream_ptr()))


def to_device(a: np.ndarray, cfg, device="cuda", io_f32: bool = False) -> torch.Tensor:
    dt = torch.float32 if io_f32 else act_dtype(cfg)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=dt)


def stream_flags(cfg) -> int:
    """Flags of a layer inside a residual stack: fp32 residual stream for bf16 layers."""
    from . import HYMBA_ADD_RESIDUAL, HYMBA_IO_F32
    return HYMBA_ADD_RESIDUAL | (HYMBA_IO_F32 if cfg.dtype == HYMBA_BF16 else 0)


class DeviceMLP:
    """The block MLP's weights in device memory and their C struct."""

    def __init__(self, cfg, w: Dict[str, np.ndarray], device="cuda"):
        from . import hymba_mlp_weights
        self.cfg = cfg
        self.c = cfg_struct(cfg)
        self.d_ff = w["w_gate"].shape[0]
        adt = act_dtype(cfg)
        self.t = {n: torch.from_numpy(np.ascontiguousarray(w[n], dtype=np.float32)).to(
            device=device, dtype=torch.float32 if n == "norm_w" else adt) for n in ("norm_w", "w_gate", "w_up", "w_down")}
        self.s = hymba_mlp_weights(*[self.t[n].data_ptr() for n in ("norm_w", "w_gate", "w_up", "w_down")])


def mlp_workspace(mlp: DeviceMLP, rows: int, device="cuda") -> torch.Tensor:
    from . import hymba_mlp_workspace_bytes
    n = hymba_mlp_workspace_bytes(ctypes.byref(mlp.c), mlp.d_ff, rows)
    if n == 0:
        raise ValueError("invalid MLP configuration")
    return torch.empty(n, dtype=torch.uint8, device=device)


def mlp(m: DeviceMLP, h: torch.Tensor, ws: torch.Tensor) -> None:
    """h += MLP(RMSNorm(h)) in place on every row of the fp32 stream h."""
    from . import hymba_mlp
    assert h.dtype == torch.float32 and h.is_contiguous()
    rows = h.numel() // m.cfg.d_model
    check(hymba_mlp(ctypes.byref(m.c), m.d_ff, ctypes.byref(m.s), h.data_ptr(), rows, ws.data_ptr(), ws.numel(),
                    current_stream_ptr()))
