"""Seeded synthetic inputs for the Hymba hybrid-head mixer.

This module is shared by the CPU oracle, the tests and the benchmark. It holds
no arithmetic of the mixer itself: it only draws random numbers with numpy's
PCG64 generator (reproducible on any machine) and rounds them to the storage
type of the layer (bf16 or fp32), so that every consumer sees identical values.

Value recipe (Hymba-1.5B shapes from the 51cto article "Hymba-1.5B", section 2
"模型架构非常巧妙": d_model 1600, 25 attention heads, 16 SSM states, GQA, RoPE;
the distributions are those of the synthetic workloads):

* X ~ N(0, 1); projection weights ~ N(0, 1/fan_in) (the second argument of N is a
  variance); meta tokens ~ N(0, 0.02).
* A_log = log(u), u ~ Uniform[1, 16] continuous, iid per (channel, state) (per SSM
  head in the SSD form).
* dt bias b = softplus^-1(dt), dt = exp(Uniform[ln 1e-3, ln 1e-1]) per channel (per
  SSM head in the SSD form).
* conv taps ~ N(0, 1/d_conv), conv bias 0; D = 1; RMSNorm gains 1; beta1 = beta2 = 1.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class LayerCfg:
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    v_head_dim: int
    d_inner: int
    d_state: int
    d_conv: int
    dt_rank: int
    n_meta: int
    window: int            # <= 0: global (full causal) attention
    is_kv_producer: int    # 1: computes its own K/V; 0: reads a producer's K/V
    dtype: int             # F32 or BF16 (activations and big weights)
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    fusion: int = 0        # 0: beta-average of the two branches; 1: concatenation [Mamba | Attention]
    ssm_heads: int = 0     # 0: A per (channel, state), Delta per channel; > 0: SSD form, A a scalar
                           # per SSM head and Delta per head (head dim d_inner / ssm_heads)

    @property
    def n_dt(self) -> int:
        """Rows of W_dt (and entries of b_dt): one per channel, or one per SSM head."""
        return self.ssm_heads if self.ssm_heads > 0 else self.d_inner

    @property
    def u_width(self) -> int:
        """Width of the fused branches (the input of W_o)."""
        return self.d_inner + self.n_q_heads * self.v_head_dim if self.fusion == 1 else self.d_inner

    @property
    def n_in(self) -> int:
        """Width of the fused input projection: [Q | K | V | x | z | B | C | dt_low]."""
        kv = self.n_kv_heads * (self.head_dim + self.v_head_dim) if self.is_kv_producer else 0
        return (self.n_q_heads * self.head_dim + kv + 2 * self.d_inner
                + self.dt_rank + 2 * self.d_state)

    def with_(self, **kw) -> "LayerCfg":
        return dataclasses.replace(self, **kw)


def tiny_layer_cfg() -> LayerCfg:
    return LayerCfg(d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64, v_head_dim=128,
                    d_inner=512, d_state=16, d_conv=4, dt_rank=16, n_meta=16, window=64,
                    is_kv_producer=1, dtype=F32)


def hymba15_layer_cfg(window: int = 1024, producer: int = 1) -> LayerCfg:
    return LayerCfg(d_model=1600, n_q_heads=25, n_kv_heads=5, head_dim=64, v_head_dim=128,
                    d_inner=3200, d_state=16, d_conv=4, dt_rank=100, n_meta=128,
                    window=window, is_kv_producer=producer, dtype=BF16)


# Workloads, named by what they are.
WORKLOADS: Dict[str, dict] = {
    # tiny fp32 layer: B=1, T=256 + 16 meta, window 64
    "tiny_f32_b1_t256": dict(kind="prefill", cfg=tiny_layer_cfg(), B=1, T=256, seed=0),
    # Hymba-1.5B-shaped SWA layer: B=1, T=2048 + 128 meta, window 1024
    "hymba15_swa1024_b1_t2048": dict(kind="prefill", cfg=hymba15_layer_cfg(1024), B=1, T=2048, seed=1),
    # the same shape as a global layer: B=4, T=8192 + 128 meta
    "hymba15_global_b4_t8192": dict(kind="prefill", cfg=hymba15_layer_cfg(0), B=4, T=8192, seed=2),
    # decode step of a KV-sharing layer pair: B=64, prompt 4096 + 128 meta, ring 1024
    "hymba15_decode_pair_b64_p4096": dict(kind="decode_pair", cfg=hymba15_layer_cfg(1024), B=64,
                                          T=4096, seed=3),
    # the SWA layer with the Mamba heads in the SSD form (50 heads of 64 channels), at the
    # stack's batch: B=8, T=4096 + 128 meta
    "hymba15_ssd_swa1024_b8_t4096": dict(kind="prefill", cfg=hymba15_layer_cfg(1024).with_(ssm_heads=50), B=8,
                                         T=4096, seed=5),
    # 32-layer mixer stack: B=8, T=4096 + 128 meta; layers 0/15/31 global; pairs share KV
    "hymba15_stack32_b8_t4096": dict(kind="stack", cfg=hymba15_layer_cfg(1024), B=8, T=4096,
                                     seed=4, n_layers=32, global_layers=(0, 15, 31)),
}


def stack_layer_cfgs(base: LayerCfg, n_layers: int, global_layers) -> List[LayerCfg]:
    """Layer configs of a KV-sharing stack: pairs (2i, 2i+1), even layers produce."""
    out = []
    for l in range(n_layers):
        w = 0 if l in global_layers else base.window
        out.append(base.with_(window=w, is_kv_producer=1 if l % 2 == 0 else 0))
    return out


def round_bf16(a) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float32."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    u = ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def to_storage(a, dtype: int) -> np.ndarray:
    """Values as stored on the device (float32 array holding bf16- or fp32-exact values)."""
    return round_bf16(a) if dtype == BF16 else np.ascontiguousarray(a, dtype=np.float32)


def _rng(*tags) -> np.random.Generator:
    return np.random.default_rng([int(t) for t in tags])


def _normal(rng, shape, var):
    return rng.standard_normal(shape) * np.sqrt(var)


def layer_weights(cfg: LayerCfg, seed: int) -> Dict[str, np.ndarray]:
    """Random-init weights of one mixer layer, as float32 arrays of storage-exact values.

    Big matrices follow the [out, in] convention: w_in [n_in, d_model],
    w_dt [n_dt, dt_rank], w_out [d_model, d_inner]. A_log is [d_inner, d_state], or
    [ssm_heads] in the SSD form.
    """
    d, di, N, r = cfg.d_model, cfg.d_inner, cfg.d_state, cfg.dt_rank
    H, G, dh, dv = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
    # row blocks of w_in in projection order; each block draws from its own stream
    blocks = [("q", H * dh, 0), ("k", G * dh, 1), ("v", G * dv, 2), ("x", di, 3), ("z", di, 4),
              ("B", N, 6), ("C", N, 7), ("dtl", r, 5)]
    rows = []
    for name, width, tag in blocks:
        blk = _normal(_rng(seed, 1, tag), (width, d), 1.0 / d)
        if name in ("k", "v") and not cfg.is_kv_producer:
            continue
        rows.append(blk)
    w_in = np.concatenate(rows, axis=0)
    nd = cfg.n_dt
    dt = np.exp(_rng(seed, 2).uniform(np.log(1e-3), np.log(1e-1), size=nd))
    a_shape = (cfg.ssm_heads,) if cfg.ssm_heads > 0 else (di, N)
    w = {
        "w_in": to_storage(w_in, cfg.dtype),
        "w_dt": to_storage(_normal(_rng(seed, 3), (nd, r), 1.0 / r), cfg.dtype),
        "b_dt": np.log(np.expm1(dt)).astype(np.float32),
        "conv_w": _normal(_rng(seed, 4), (di, cfg.d_conv), 1.0 / cfg.d_conv).astype(np.float32),
        "conv_b": np.zeros(di, np.float32),
        "A_log": np.log(_rng(seed, 5).uniform(1.0, 16.0, size=a_shape)).astype(np.float32),
        "D": np.ones(di, np.float32),
        "norm_attn_w": np.ones(H * dv, np.float32),
        "norm_ssm_w": np.ones(di, np.float32),
        "beta1": np.ones(H * dv, np.float32),
        "beta2": np.ones(di, np.float32),
        "w_out": to_storage(_normal(_rng(seed, 6), (d, cfg.u_width), 1.0 / cfg.u_width), cfg.dtype),
        "meta": to_storage(_normal(_rng(seed, 7), (cfg.n_meta, d), 0.02), cfg.dtype),
    }
    return w


def layer_input(cfg: LayerCfg, B: int, T: int, seed: int, tag: int = 0) -> np.ndarray:
    """User-token input X ~ N(0, 1), [B, T, d_model], storage-exact float32."""
    return to_storage(_rng(seed, 100, tag).standard_normal((B, T, cfg.d_model)), cfg.dtype)


def perturbed_weights(w: Dict[str, np.ndarray], cfg: LayerCfg, seed: int,
                      scale: float = 0.5) -> Dict[str, np.ndarray]:
    """Copy of w with the per-channel parameters (conv bias, D, gains, betas) drawn away
    from their defaults, so that tests exercise every term of the layer."""
    out = dict(w)
    di = cfg.d_inner
    g = _rng(seed, 9)
    out["conv_b"] = (g.standard_normal(di) * 0.2).astype(np.float32)
    out["D"] = (1.0 + g.standard_normal(di) * scale).astype(np.float32)
    out["norm_attn_w"] = (1.0 + g.standard_normal(w["norm_attn_w"].shape) * scale).astype(np.float32)
    out["norm_ssm_w"] = (1.0 + g.standard_normal(di) * scale).astype(np.float32)
    out["beta1"] = (1.0 + g.standard_normal(w["beta1"].shape) * scale).astype(np.float32)
    out["beta2"] = (1.0 + g.standard_normal(di) * scale).astype(np.float32)
    return out


def workload(name: str) -> dict:
    return dict(WORKLOADS[name])


def affine_kv(cfg: LayerCfg, seed: int, spread: float = 0.5) -> Dict[str, np.ndarray]:
    """Weights of a secondary layer's affine adaptation of shared K and V, as two
    [G*dh + G*dv] fp32 vectors (the G K vectors, then the G V vectors): scales
    ~ Uniform[1 - spread, 1 + spread], biases ~ N(0, 0.1^2). The pages give no
    initialisation; these keep every term of the transform visible in a test."""
    G, dh, dv = cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
    g = _rng(seed, 11)
    n = G * (dh + dv)
    return {"kv_scale": g.uniform(1.0 - spread, 1.0 + spread, size=n).astype(np.float32),
            "kv_bias": (g.standard_normal(n) * 0.1).astype(np.float32)}


def mlp_weights(d_model: int, d_ff: int, dtype: int, seed: int) -> Dict[str, np.ndarray]:
    """The block's MLP: W_gate, W_up [d_ff, d_model] ~ N(0, 1/d_model), W_down [d_model, d_ff]
    ~ N(0, 1/d_ff) (storage-exact), and its pre-norm gain (1)."""
    return {"norm_w": np.ones(d_model, np.float32),
            "w_gate": to_storage(_normal(_rng(seed, 21), (d_ff, d_model), 1.0 / d_model), dtype),
            "w_up": to_storage(_normal(_rng(seed, 22), (d_ff, d_model), 1.0 / d_model), dtype),
            "w_down": to_storage(_normal(_rng(seed, 23), (d_model, d_ff), 1.0 / d_ff), dtype)}


def with_pre_norm(w: Dict[str, np.ndarray], cfg: LayerCfg, seed: int = 0, scale: float = 0.0) -> Dict[str, np.ndarray]:
    """A copy of the mixer weights with the block's pre-mixer RMSNorm gain (1, or 1 + N(0, scale^2))."""
    g = np.ones(cfg.d_model) + (_rng(seed, 24).standard_normal(cfg.d_model) * scale if scale else 0.0)
    return dict(w, pre_norm_w=g.astype(np.float32))


HYMBA15_D_FF = 5504  # MLP intermediate size of Hymba-1.5B (51cto article, section 2)
