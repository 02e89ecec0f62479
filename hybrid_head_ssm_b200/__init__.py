"""Python binding of libhymba.so, the B200 Hymba hybrid-head mixer.

Argument marshalling only: the structs of include/hymba.h as ctypes structures and
the exported functions under the same names. Every step of the mixer runs in the
library's CUDA kernels; there is no Python or CPU fallback. Importing this package
fails loudly when the library has not been built.

PyTorch is used only by the helpers at the bottom (`weights_struct`, `kv_struct`,
...) to hand device pointers and the current stream to the library.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhymba.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python hybrid_head_ssm_b200/build.py` "
        "(the mixer has no non-CUDA implementation)")

_lib = ctypes.CDLL(LIB_PATH)

HYMBA_OK = 0
HYMBA_ERR_INVALID_ARG = -1
HYMBA_ERR_UNSUPPORTED = -2
HYMBA_ERR_WORKSPACE_TOO_SMALL = -3
HYMBA_ERR_KV_INCOMPATIBLE = -4
HYMBA_ERR_CUDA = -5
HYMBA_ERR_DEVICE_TIMEOUT = -6
HYMBA_ERR_DEVICE_RANGE = -7
HYMBA_ERR_SCRATCH_LIMIT = -8

HYMBA_F32 = 0
HYMBA_BF16 = 1
HYMBA_F16 = 2
HYMBA_X_HAS_META = 1
HYMBA_ADD_RESIDUAL = 2
HYMBA_IO_F32 = 4
HYMBA_PRE_NORM = 8
HYMBA_FUSION_AVERAGE = 0
HYMBA_FUSION_CONCAT = 1
HYMBA_MODE_PREFILL = 0
HYMBA_MODE_DECODE = 1

_i32, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class hymba_layer_cfg(ctypes.Structure):
    _fields_ = [("d_model", _i32), ("n_q_heads", _i32), ("n_kv_heads", _i32), ("head_dim", _i32),
                ("v_head_dim", _i32), ("d_inner", _i32), ("d_state", _i32), ("d_conv", _i32),
                ("dt_rank", _i32), ("n_meta", _i32), ("window", _i32), ("is_kv_producer", _i32),
                ("dtype", _i32), ("rope_base", _f32), ("rms_eps", _f32), ("fusion", _i32),
                ("ssm_heads", _i32)]


class hymba_layer_weights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("w_in", "w_dt", "b_dt", "conv_w", "conv_b", "A_log", "D",
                                   "norm_attn_w", "norm_ssm_w", "beta1", "beta2", "w_out", "meta",
                                   "kv_scale", "kv_bias", "pre_norm_w")]


class hymba_kv(ctypes.Structure):
    _fields_ = [("k_seq", _vp), ("v_seq", _vp), ("seq_cap", _i32), ("k_cache", _vp), ("v_cache", _vp),
                ("len", _vp), ("cache_cap", _i32), ("batch", _i32), ("n_meta", _i32),
                ("n_kv_heads", _i32), ("head_dim", _i32), ("v_head_dim", _i32), ("dtype", _i32),
                ("window", _i32)]


class hymba_mlp_weights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("norm_w", "w_gate", "w_up", "w_down")]


class hymba_ssm_state(ctypes.Structure):
    _fields_ = [("h", _vp), ("conv", _vp)]


_P = ctypes.POINTER
_sig = {
    "hymba_mixer_prefill": (ctypes.c_int, [_P(hymba_layer_cfg), _P(hymba_layer_weights), _vp, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, _vp, _P(hymba_kv), _P(hymba_ssm_state),
                                           _vp, _sz, _vp]),
    "hymba_mixer_decode": (ctypes.c_int, [_P(hymba_layer_cfg), _P(hymba_layer_weights), _vp, ctypes.c_int,
                                          ctypes.c_int, _vp, _P(hymba_kv), _P(hymba_ssm_state), _vp, _sz, _vp]),
    "hymba_kv_share": (ctypes.c_int, [_P(hymba_kv), _P(hymba_layer_cfg), _P(hymba_kv)]),
    "hymba_mlp": (ctypes.c_int, [_P(hymba_layer_cfg), ctypes.c_int, _P(hymba_mlp_weights), _vp, ctypes.c_longlong,
                                 _vp, _sz, _vp]),
    "hymba_mlp_workspace_bytes": (_sz, [_P(hymba_layer_cfg), ctypes.c_int, ctypes.c_longlong]),
    "hymba_workspace_bytes": (_sz, [_P(hymba_layer_cfg), ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "hymba_workspace_layout": (ctypes.c_int, [_P(hymba_layer_cfg), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              _P(ctypes.c_int64), ctypes.c_int]),
    "hymba_cache_bytes": (_sz, [_P(hymba_layer_cfg), ctypes.c_int, ctypes.c_int]),
    "hymba_kv_bytes": (ctypes.c_uint64, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int64, ctypes.c_int, ctypes.c_int]),
    "hymba_ssm_state_bytes": (ctypes.c_uint64, [ctypes.c_int] * 5),
    "hymba_get_device_status": (ctypes.c_int, [_vp]),
    "hymba_get_device_diag": (ctypes.c_int, [_P(ctypes.c_int32), ctypes.c_int]),
    "hymba_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "hymba_trace_enable": (ctypes.c_int, [ctypes.c_int]),
    "hymba_trace_collect": (ctypes.c_int, [_P(ctypes.c_char_p), _P(ctypes.c_float), ctypes.c_int]),
    "hymba_trace_only": (ctypes.c_int, [ctypes.c_char_p]),
    "hymba_launch_count": (ctypes.c_uint64, []),
    "hymba_attn_decode_static": (ctypes.c_int, [_P(hymba_layer_cfg), _vp, ctypes.c_int64, _P(hymba_kv), _vp,
                                                ctypes.c_int, _vp]),
    "hymba_probe_unit_rates": (ctypes.c_int, [_P(ctypes.c_double), ctypes.c_int, _vp]),
    "hymba_debug_set_wait_limit": (ctypes.c_int, [ctypes.c_longlong]),
    "hymba_debug_stalled_wait": (ctypes.c_int, [_vp]),
}
EXPORTS = tuple(_sig)

for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
    globals()[_name] = _fn


class HymbaError(RuntimeError):
    pass


def check(rc: int) -> int:
    """Raise HymbaError for a negative status code."""
    if rc < 0:
        raise HymbaError(f"hymba error {rc}: {hymba_strerror(rc).decode()}")
    return rc


def workspace_layout(cfg: hymba_layer_cfg, B: int, T: int, mode: int) -> dict:
    out = (ctypes.c_int64 * 10)()
    check(hymba_workspace_layout(ctypes.byref(cfg), B, T, mode, out, 10))
    keys = ("total", "P", "ldP", "delta", "O", "ypre", "U", "rope", "part", "n_split")
    return dict(zip(keys, list(out)))


def unit_rates():
    """Measured exp2 (fp32, fp16 pairs) and fp32 FMA results per clock per SM."""
    out = (ctypes.c_double * 3)()
    check(hymba_probe_unit_rates(out, 3, current_stream_ptr()))
    return {"ex2_f32": out[0], "ex2_f16x2": out[1], "ffma_f32": out[2]}


def device_diag():
    out = (ctypes.c_int32 * 7)()
    check(hymba_get_device_diag(out, 7))
    return list(out)


def trace_collect(max_records: int = 8192):
    names = (ctypes.c_char_p * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = check(hymba_trace_collect(names, ms, max_records))
    return [(names[i].decode(), ms[i]) for i in range(n)]


# ---------------------------------------------------------------------------
# helpers that marshal torch tensors (device memory) into the structs
# ---------------------------------------------------------------------------

def cfg_struct(c) -> hymba_layer_cfg:
    """From any object with the hymba_layer_cfg field names (e.g. synth.LayerCfg)."""
    return hymba_layer_cfg(*[getattr(c, n) for n, _ in hymba_layer_cfg._fields_])


def _ptr(t):
    return None if t is None else t.data_ptr()


def weights_struct(w: dict) -> hymba_layer_weights:
    """From a dict of device tensors named like the struct fields."""
    return hymba_layer_weights(*[_ptr(w.get(n)) for n, _ in hymba_layer_weights._fields_])


def kv_dtype_code(cfg) -> int:
    """K/V element type of a layer: fp16 for bf16 layers, fp32 for fp32 layers."""
    return HYMBA_F16 if cfg.dtype == HYMBA_BF16 else HYMBA_F32


def kv_struct(cfg, batch: int, k_seq=None, v_seq=None, k_cache=None, v_cache=None, length=None) -> hymba_kv:
    return hymba_kv(k_seq=_ptr(k_seq), v_seq=_ptr(v_seq),
                    seq_cap=0 if k_seq is None else k_seq.shape[2],
                    k_cache=_ptr(k_cache), v_cache=_ptr(v_cache), len=_ptr(length),
                    cache_cap=0 if k_cache is None else k_cache.shape[2], batch=batch,
                    n_meta=cfg.n_meta, n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                    v_head_dim=cfg.v_head_dim, dtype=kv_dtype_code(cfg), window=cfg.window)


def state_struct(h=None, conv=None) -> hymba_ssm_state:
    return hymba_ssm_state(h=_ptr(h), conv=_ptr(conv))


def current_stream_ptr():
    import torch
    return torch.cuda.current_stream().cuda_stream
