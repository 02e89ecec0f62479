"""Plain fp64 CPU oracle of the Hymba parallel hybrid-head mixer.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline may import this module. The product (the CUDA library and its Python
binding) never calls it, and it shares no code with the product: the only module
both sides use is `synth`, which draws the seeded inputs.

Everything is computed in float64 with straight loops and library matmuls, in
the order the pages give the steps. Sources, cited by page title and section:

* [Hymba Guide] "Hymba Guide: NVIDIA Hybrid-Head Mamba & Attention SLM":
  section "Parallel Hybrid-Head Layer Formulation" (attention heads and Mamba heads
  run in parallel on one input, then one output projection W_o), "Learnable
  Meta-Tokens" (X_input = [M_1..M_k, x_1..x_T]; meta tokens pre-populate the SSM
  state and are attended by every token), "Cross-Layer KV Cache Sharing"
  (secondary layers reuse the primary layer's K, V without new buffers).
* [Jamba] "Jamba: Hybrid SSM-Transformer", "How It Actually Works" section 1: the
  selective scan h_t = exp(Delta_t A) h_{t-1} + (Delta_t B_t) x_t, y_t = C_t h_t,
  and Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V with MHA or GQA; section 2
  and "Worked Example": the KV-cache size formula.
* [Lecture 04] "Lecture 04 - Beyond the Dense Transformer: Mamba, SSMs, and the
  Hybrid Wave": section 1 (the KV cache grows by one K, V per token), section 2
  (fixed-size SSM state; Delta_t -> 0 leaves the state unchanged, large Delta_t
  resets it; A_bar = exp(Delta A), B_bar ~ Delta B), section 3 (the scan equals a
  masked semiseparable matrix product), section 8 (kv_cache_gb, ssm_state_gb).
* [51cto] the 51cto article on Hymba-1.5B, section 2 "模型架构非常巧妙": GQA and
  RoPE, sliding-window attention in most layers with 3 full-attention layers,
  KV shared between pairs of layers.

Readings taken where the pages are silent:

* Fusion of the two branches: each branch is RMS-normalised over its full
  width, scaled per channel by beta1 / beta2, and the two are averaged before
  W_o; averaging needs equal widths, so the V head dim is d_inner / n_q_heads.
  The [Hymba Guide] formula concatenates instead: that variant (cfg.fusion = 1)
  places the same normalised, beta-scaled branches side by side, Mamba first, with
  the V head dim equal to the Q/K head dim, and W_o takes d_inner + n_q_heads *
  v_head_dim inputs.
* One input projection yields [Q | K | V | x | z | B | C | dt_low] in that order.
  A consumer (KV-sharing secondary) layer has no K, V rows.
* A consumer's affine adaptation of the shared K, V acts on the K that is shared
  (after RoPE) and on V, per KV head and dimension, with its own scale and bias
  for each; a consumer without those weights shares K and V unchanged.
* RoPE is rotate-half with theta_i = base^(-2i/head_dim); meta tokens take
  positions 0..m-1 and user token t takes m + t; K is kept after RoPE.
* Key j is visible to query i iff j <= i and (j < m or i - j < W); W <= 0 is
  global. So the window counts non-meta keys including the query itself.
* The Mamba branch: depthwise causal conv (zero history before the first meta
  row) + bias, SiLU; Delta = softplus(dt_low W_dt^T + b_dt); A = -exp(A_log);
  y = (C_t . h_t + D x_t) * SiLU(z_t) with x_t the conv output.
* The SSD form of the Mamba heads ([Lecture 04] section 3 names it without
  formulas; cfg.ssm_heads > 0): the channels split into ssm_heads heads of
  d_inner / ssm_heads consecutive channels; W_dt, b_dt and A_log have one entry per
  head, so Delta_t and A are scalars per head shared by its channels and all states;
  conv, B_t, C_t, D and the gate are as in the selective form.
* The block around the mixer ([51cto] section 2 gives the MLP intermediate size 5504
  and nothing else): pre-norm residual blocks, h + Mixer(RMSNorm(h)) then
  h + MLP(RMSNorm(h)), each RMSNorm with its own gain, and a SiLU-gated MLP
  W_down (SiLU(W_gate n) * W_up n) as in the Llama-family blocks the model builds on.
* The decode cache holds the meta block in slots 0..m-1 and the non-meta
  positions in a ring: position p >= m lives in slot m + (p - m) mod R, R = cap - m.
  The conv state holds the last d_conv pre-conv inputs, oldest first.

Parity pins (tests/test_oracle_*.py): sequential-vs-semiseparable scan, Delta->0
and Delta-large limits, a hand-worked single step, brute-force per-query softmax
loops, window >= T equals full causal, meta visibility, GQA equals repeated KV,
RoPE relative invariance, conv impulse response and causality, RMSNorm scale
invariance, beta2 = 0, decode-by-decode equals prefill (across ring wrap), and the
pages' printed cache sizes, RMSNorm's epsilon inside the square root, and the
decode-state byte count against the arrays a decode step actually carries.

Parity unpinned (no page value can check it, and none of the pins above would
notice a change of it): the order of the row blocks of the fused projection
[Q | K | V | x | z | B | C | dt_low] is a layout reading, not arithmetic (B and C
sit before dt_low so that their columns start on 16-byte boundaries); and the
whole-layer composition of the pinned steps (the fusion reading) has no page value
to check against beyond the invariants above.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# elementwise functions
# ----------------------------------------------------------------------------

def silu(u: np.ndarray) -> np.ndarray:
    """SiLU(u) = u / (1 + exp(-u))."""
    return u / (1.0 + np.exp(-u))


def softplus(u: np.ndarray) -> np.ndarray:
    """softplus(u) = log(1 + exp(u)), evaluated without overflow."""
    return np.logaddexp(0.0, u)


# ----------------------------------------------------------------------------
# attention branch
# ----------------------------------------------------------------------------

def rope(v: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotary position embedding ([51cto] section 2 names RoPE), rotate-half form.

    v: [..., L, dh]; pos: [L] absolute positions. Pair (i, i + dh/2) is rotated by
    the angle pos * base^(-2i/dh).
    """
    dh = v.shape[-1]
    half = dh // 2
    theta = base ** (-2.0 * np.arange(half, dtype=np.float64) / dh)
    ang = pos.astype(np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def key_visible(i: int, j: int, n_meta: int, window: int) -> bool:
    """Visibility of key position j to query position i (meta prefix + window)."""
    if j > i:
        return False
    if j < n_meta or window <= 0:
        return True
    return i - j < window


def visibility_mask(q_pos: np.ndarray, k_pos: np.ndarray, n_meta: int, window: int) -> np.ndarray:
    """Boolean [Lq, Lk] mask: the rule of key_visible applied to every pair."""
    i = np.asarray(q_pos)[:, None]
    j = np.asarray(k_pos)[None, :]
    in_span = (j < n_meta) | (i - j < window) if window > 0 else np.ones_like(j >= 0)
    return (j <= i) & in_span


def gqa_group(h: int, n_q_heads: int, n_kv_heads: int) -> int:
    """KV head read by query head h: consecutive query heads share one KV head."""
    return h // (n_q_heads // n_kv_heads)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """softmax(Q K^T / sqrt(d_k) + mask) V per query head, GQA ([Jamba] section 1).

    q [H, Lq, dh], k [G, Lk, dh], v [G, Lk, dv], mask [Lq, Lk] -> [H, Lq, dv].
    """
    H, G = q.shape[0], k.shape[0]
    out = np.zeros((H, q.shape[1], v.shape[2]))
    scale = 1.0 / math.sqrt(q.shape[2])
    for h in range(H):
        g = gqa_group(h, H, G)
        s = (q[h] @ k[g].T) * scale
        s = np.where(mask, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[h] = p @ v[g]
    return out


def adapt_shared_kv(k: np.ndarray, v: np.ndarray, w: Dict[str, np.ndarray], G: int, dh: int, dv: int):
    """The secondary layer's head-specific affine adaptation of shared K and V
    ([Hymba Guide] "Cross-Layer KV Cache Sharing", section 1: K~ = K * w_scale + b_bias,
    elementwise, per KV head; V takes the same form with its own scale and bias).

    k [G, L, dh], v [G, L, dv]; w["kv_scale"], w["kv_bias"] [G*dh + G*dv]: the G K
    vectors (dh each) first, then the G V vectors (dv each). Without those weights the
    layer shares K and V unchanged.
    """
    if w.get("kv_scale") is None:
        return k, v
    s = np.asarray(w["kv_scale"], dtype=np.float64)
    b = np.asarray(w["kv_bias"], dtype=np.float64)
    nk = G * dh
    ks, kb = s[:nk].reshape(G, 1, dh), b[:nk].reshape(G, 1, dh)
    vs, vb = s[nk:].reshape(G, 1, dv), b[nk:].reshape(G, 1, dv)
    return k * ks + kb, v * vs + vb


# ----------------------------------------------------------------------------
# Mamba branch
# ----------------------------------------------------------------------------

def causal_conv(x: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Depthwise causal conv: out[t, c] = b[c] + sum_k w[c, k] * x[t - (K-1) + k, c].

    x [L, C]; w [C, K]; inputs before t = 0 are zero (the sequence starts at the
    first meta row; a decode step carries its own conv state instead).
    """
    L, C = x.shape
    K = w.shape[1]
    xp = np.concatenate([np.zeros((K - 1, C)), x], axis=0)
    out = np.tile(b.astype(np.float64), (L, 1))
    for k in range(K):
        out += w[:, k][None, :] * xp[k:k + L]
    return out


def selective_scan(xc: np.ndarray, delta: np.ndarray, A: np.ndarray, Bm: np.ndarray,
                   Cm: np.ndarray, D: np.ndarray, h0: Optional[np.ndarray] = None
                   ) -> Tuple[np.ndarray, np.ndarray]:
    """Selective scan, one step per token ([Jamba] section 1, [Lecture 04] section 2):

        h_t = exp(Delta_t A) * h_{t-1} + (Delta_t B_t) x_t,   y_t = C_t . h_t + D x_t

    xc, delta [L, C]; A [C, N]; Bm, Cm [L, N]; D [C]; h0 [C, N] or zeros.
    Returns (y [L, C] before the gate, h_L [C, N]).
    """
    L, C = xc.shape
    h = np.zeros((C, A.shape[1])) if h0 is None else h0.astype(np.float64).copy()
    y = np.zeros((L, C))
    for t in range(L):
        dA = np.exp(delta[t][:, None] * A)
        dBx = (delta[t] * xc[t])[:, None] * Bm[t][None, :]
        h = dA * h + dBx
        y[t] = h @ Cm[t] + D * xc[t]
    return y, h


def ssm_params(cfg, w: Dict[str, np.ndarray], dtl: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Delta [L, d_inner] and A [d_inner, N] of the scan from the dt_low rows [L, r].

    Delta = softplus(dt_low W_dt^T + b_dt) and A = -exp(A_log). In the selective form
    (cfg.ssm_heads == 0) both are per channel, A per (channel, state). In the SSD form
    ([Lecture 04] section 3: Mamba-2 makes A a scalar times the identity and adds a
    multi-head structure) W_dt, b_dt and A_log have one entry per SSM head: the head's
    Delta_t and scalar A serve its d_inner / ssm_heads consecutive channels and all N
    states, so the same recurrence applies with those values repeated.
    """
    delta = softplus(dtl @ w["w_dt"].T + w["b_dt"])
    A = -np.exp(w["A_log"])
    nh = getattr(cfg, "ssm_heads", 0)
    if nh > 0:
        P = cfg.d_inner // nh
        delta = np.repeat(delta, P, axis=-1)
        A = np.repeat(A, P)[:, None] * np.ones((1, cfg.d_state))
    return delta, A


# ----------------------------------------------------------------------------
# fusion
# ----------------------------------------------------------------------------

def rms_norm(a: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """gain * a / sqrt(mean(a^2) + eps), the mean over the last axis."""
    return gain * a / np.sqrt(np.mean(a * a, axis=-1, keepdims=True) + eps)


def fuse(o_attn: np.ndarray, y_ssm: np.ndarray, w: Dict[str, np.ndarray], eps: float) -> np.ndarray:
    """U = (beta1 * RMS(attn) + beta2 * RMS(ssm)) / 2 (both [L, d_inner])."""
    a = rms_norm(o_attn, w["norm_attn_w"].astype(np.float64), eps)
    s = rms_norm(y_ssm, w["norm_ssm_w"].astype(np.float64), eps)
    return (w["beta1"].astype(np.float64) * a + w["beta2"].astype(np.float64) * s) / 2.0


def fuse_concat(o_attn: np.ndarray, y_ssm: np.ndarray, w: Dict[str, np.ndarray], eps: float) -> np.ndarray:
    """U = Concat[beta2 * RMS(ssm), beta1 * RMS(attn)] ([Hymba Guide] "Parallel Hybrid-Head
    Layer Formulation": y = W_o(Concat[MambaHeads(x), AttentionHeads(x)]), the Mamba heads
    first). Each branch keeps its RMSNorm and beta scaling; the branches are placed side
    by side instead of averaged, so they may differ in width (ssm [L, d_inner], attn
    [L, n_q_heads * v_head_dim]) and W_o takes both widths."""
    a = rms_norm(o_attn, w["norm_attn_w"].astype(np.float64), eps) * w["beta1"].astype(np.float64)
    s = rms_norm(y_ssm, w["norm_ssm_w"].astype(np.float64), eps) * w["beta2"].astype(np.float64)
    return np.concatenate([s, a], axis=-1)


def fuse_layer(cfg, o_attn, y_ssm, w, eps):
    """The layer's fusion: the beta-average, or the concatenation when cfg.fusion == 1."""
    return fuse_concat(o_attn, y_ssm, w, eps) if getattr(cfg, "fusion", 0) == 1 else fuse(o_attn, y_ssm, w, eps)


# ----------------------------------------------------------------------------
# the layer
# ----------------------------------------------------------------------------

def split_projection(cfg, p: np.ndarray) -> Dict[str, np.ndarray]:
    """Split the fused projection [L, n_in] into its named blocks."""
    H, G, dh, dv = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
    widths = [("q", H * dh)]
    if cfg.is_kv_producer:
        widths += [("k", G * dh), ("v", G * dv)]
    widths += [("x", cfg.d_inner), ("z", cfg.d_inner), ("B", cfg.d_state), ("C", cfg.d_state),
               ("dtl", cfg.dt_rank)]
    out, c = {}, 0
    for name, wd in widths:
        out[name] = p[:, c:c + wd]
        c += wd
    assert c == p.shape[1]
    return out


def _f64(w: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    return {k: (None if v is None else np.asarray(v, dtype=np.float64)) for k, v in w.items()}


def mixer_prefill_row(cfg, w: Dict[str, np.ndarray], x: np.ndarray,
                      kv_shared: Optional[Tuple[np.ndarray, np.ndarray]] = None,
                      residual: bool = False, x_has_meta: bool = False):
    """One sequence through the mixer layer.

    x [T, d_model] user tokens, or [T', d_model] rows that already start with the
    meta rows (x_has_meta, the input of a later layer of a stack). Returns dict
    with y [T', d_model] (meta rows included), k [G, T', dh], v [G, T', dv] (the
    producer's, or the shared ones), h [d_inner, N] and conv [d_inner, K] (final
    decode state).
    """
    w = _f64(w)
    m = cfg.n_meta
    H, G, dh, dv, di = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim, cfg.d_inner
    if x_has_meta:
        xh = x.astype(np.float64)
    else:
        # meta tokens prepended ([Hymba Guide] "Learnable Meta-Tokens")
        xh = np.concatenate([w["meta"], x.astype(np.float64)], axis=0)
    Tp = xh.shape[0]
    # one projection for both head families ([Hymba Guide] "Parallel Hybrid-Head Layer")
    blocks = split_projection(cfg, xh @ w["w_in"].T)
    pos = np.arange(Tp)
    q = rope(blocks["q"].reshape(Tp, H, dh).transpose(1, 0, 2), pos, cfg.rope_base)
    if cfg.is_kv_producer:
        k = rope(blocks["k"].reshape(Tp, G, dh).transpose(1, 0, 2), pos, cfg.rope_base)
        v = blocks["v"].reshape(Tp, G, dv).transpose(1, 0, 2)
    else:
        k, v = (np.asarray(a, dtype=np.float64) for a in kv_shared)
    # a secondary layer adapts the shared K, V ([Hymba Guide] Cross-Layer KV Cache Sharing)
    ka, va = (k, v) if cfg.is_kv_producer else adapt_shared_kv(k, v, w, G, dh, dv)
    # attention heads: causal GQA over the meta prefix + window
    mask = visibility_mask(pos, pos, m, cfg.window)
    o = attention(q, ka, va, mask).transpose(1, 0, 2).reshape(Tp, H * dv)
    # Mamba heads: conv, Delta, scan, gate
    xc = silu(causal_conv(blocks["x"], w["conv_w"], w["conv_b"]))
    delta, A = ssm_params(cfg, w, blocks["dtl"])
    y_pre, h = selective_scan(xc, delta, A, blocks["B"], blocks["C"], w["D"])
    y_ssm = y_pre * silu(blocks["z"])
    # fusion and the shared output projection
    u = fuse_layer(cfg, o, y_ssm, w, cfg.rms_eps)
    y = u @ w["w_out"].T
    if residual:
        y = y + xh
    # the decode conv state: the last d_conv pre-conv inputs, oldest first, with the zero
    # history before the first row when the sequence is shorter than the conv
    K = cfg.d_conv
    xpad = np.concatenate([np.zeros((K, di)), blocks["x"]], axis=0)
    conv_state = xpad[-K:].T.copy()
    return dict(y=y, k=k, v=v, h=h, conv=conv_state, o_attn=o, y_ssm=y_ssm, u=u, delta=delta)


def mixer_prefill(cfg, w, x: np.ndarray, kv_shared=None, residual: bool = False,
                  x_has_meta: bool = False):
    """Batched prefill, x [B, T, d]; kv_shared = (k [B,G,T',dh], v [B,G,T',dv])."""
    rows = []
    for b in range(x.shape[0]):
        sh = None if kv_shared is None else (kv_shared[0][b], kv_shared[1][b])
        rows.append(mixer_prefill_row(cfg, w, x[b], sh, residual, x_has_meta))
    return {key: np.stack([r[key] for r in rows]) for key in rows[0] if rows[0][key] is not None}


# ----------------------------------------------------------------------------
# the Hymba block around the mixer ([51cto] section 2: MLP intermediate size 5504)
# ----------------------------------------------------------------------------

def mlp(h: np.ndarray, w: Dict[str, np.ndarray], eps: float) -> np.ndarray:
    """The block's pre-norm MLP with its residual: n = RMSNorm(h) * g,
    h + W_down (SiLU(W_gate n) * (W_up n)). h [L, d]; w_gate, w_up [d_ff, d]; w_down [d, d_ff]."""
    w = _f64(w)
    n = rms_norm(h.astype(np.float64), w["norm_w"], eps)
    a = silu(n @ w["w_gate"].T) * (n @ w["w_up"].T)
    return h + a @ w["w_down"].T


def block_prefill_row(cfg, w_mixer, w_mlp, h: np.ndarray, kv_shared=None):
    """One Hymba block on one sequence's stream h [T', d] (meta rows included):
    h1 = h + Mixer(RMSNorm(h) * g_pre), then h2 = MLP(h1) with its own pre-norm.
    Returns the mixer's dict with y = h2 (and h1)."""
    n = rms_norm(h.astype(np.float64), np.asarray(w_mixer["pre_norm_w"], dtype=np.float64), cfg.rms_eps)
    r = mixer_prefill_row(cfg, w_mixer, n, kv_shared, residual=False, x_has_meta=True)
    h1 = h + r["y"]
    r = dict(r, h1=h1, y=mlp(h1, w_mlp, cfg.rms_eps))
    return r


def block_prefill(cfg, w_mixer, w_mlp, h: np.ndarray, kv_shared=None):
    """Batched block_prefill_row, h [B, T', d]."""
    rows = []
    for b in range(h.shape[0]):
        sh = None if kv_shared is None else (kv_shared[0][b], kv_shared[1][b])
        rows.append(block_prefill_row(cfg, w_mixer, w_mlp, h[b], sh))
    return {key: np.stack([r[key] for r in rows]) for key in rows[0] if rows[0][key] is not None}


def block_decode(cfg, w_mixer, w_mlp, h_t: np.ndarray, cache: dict, hs: np.ndarray, conv: np.ndarray):
    """One decode step of the block: h_t [B, d] -> MLP(h_t + Mixer(RMSNorm(h_t) * g_pre))."""
    n = rms_norm(h_t.astype(np.float64), np.asarray(w_mixer["pre_norm_w"], dtype=np.float64), cfg.rms_eps)
    h1 = h_t + mixer_decode(cfg, w_mixer, n, cache, hs, conv, residual=False)
    return mlp(h1, w_mlp, cfg.rms_eps)


# ----------------------------------------------------------------------------
# decode: cache layout and one step
# ----------------------------------------------------------------------------

def ring_slot(p: int, n_meta: int, ring: int) -> int:
    """Cache slot of absolute position p: meta positions keep their own slot, the
    others wrap in a ring of `ring` slots."""
    return p if p < n_meta else n_meta + (p - n_meta) % ring


def cache_from_prefill(cfg, k: np.ndarray, v: np.ndarray, cap: int):
    """Decode cache after a prefill: k [B,G,T',dh] -> slots of a cache with `cap` slots."""
    B, G, Tp, _ = k.shape
    m = cfg.n_meta
    ring = cap - m
    kc = np.zeros((B, G, cap, k.shape[3]))
    vc = np.zeros((B, G, cap, v.shape[3]))
    for p in range(Tp):
        if p >= m and p < Tp - ring:
            continue  # overwritten by a later position
        s = ring_slot(p, m, ring)
        kc[:, :, s] = k[:, :, p]
        vc[:, :, s] = v[:, :, p]
    return dict(k=kc, v=vc, len=np.full(B, Tp, dtype=np.int64))


def mixer_decode(cfg, w, x_t: np.ndarray, cache: dict, h: np.ndarray, conv: np.ndarray,
                 residual: bool = False):
    """One decode step for every sequence of the batch.

    x_t [B, d]; cache dict(k [B,G,cap,dh], v [B,G,cap,dv], len [B]) is updated in
    place: a producer writes the new K, V at position p = len[b] and sets len = p+1;
    a consumer reads the producer's cache at p = len[b] - 1. h [B, di, N] and
    conv [B, di, K] are updated in place. Returns y_t [B, d].
    """
    w = _f64(w)
    B = x_t.shape[0]
    m = cfg.n_meta
    H, G, dh, dv, di = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim, cfg.d_inner
    cap = cache["k"].shape[2]
    ring = cap - m
    y = np.zeros((B, cfg.d_model))
    for b in range(B):
        p = int(cache["len"][b]) if cfg.is_kv_producer else int(cache["len"][b]) - 1
        blocks = split_projection(cfg, x_t[b:b + 1].astype(np.float64) @ w["w_in"].T)
        q = rope(blocks["q"].reshape(1, H, dh).transpose(1, 0, 2), np.array([p]), cfg.rope_base)
        if cfg.is_kv_producer:
            kn = rope(blocks["k"].reshape(1, G, dh).transpose(1, 0, 2), np.array([p]), cfg.rope_base)
            vn = blocks["v"].reshape(1, G, dv).transpose(1, 0, 2)
            s = ring_slot(p, m, ring)
            cache["k"][b, :, s] = kn[:, 0]
            cache["v"][b, :, s] = vn[:, 0]
            cache["len"][b] = p + 1
        # visible positions and the slots holding them
        vis = [j for j in range(p + 1) if key_visible(p, j, m, cfg.window)]
        assert all(j < m or p - j < ring for j in vis), "cache too small for the span"
        slots = [ring_slot(j, m, ring) for j in vis]
        kk = cache["k"][b][:, slots]
        vv = cache["v"][b][:, slots]
        if not cfg.is_kv_producer:
            kk, vv = adapt_shared_kv(kk, vv, w, G, dh, dv)
        o = attention(q, kk, vv, np.ones((1, len(vis)), dtype=bool)).transpose(1, 0, 2).reshape(1, H * dv)
        # Mamba step: shift the conv state, conv, Delta, one scan step
        conv[b] = np.concatenate([conv[b][:, 1:], blocks["x"].T], axis=1)
        xc = silu(w["conv_b"] + np.sum(w["conv_w"] * conv[b], axis=1))[None, :]
        delta, A = ssm_params(cfg, w, blocks["dtl"])
        y_pre, h[b] = selective_scan(xc, delta, A, blocks["B"], blocks["C"], w["D"], h[b])
        y_ssm = y_pre * silu(blocks["z"])
        u = fuse_layer(cfg, o, y_ssm, w, cfg.rms_eps)
        y[b] = (u @ w["w_out"].T)[0] + (x_t[b] if residual else 0.0)
    return y


# ----------------------------------------------------------------------------
# cache sizing ([Jamba] section 2 and "Worked Example"; [Lecture 04] section 8)
# ----------------------------------------------------------------------------

def kv_cache_bytes(n_attn_layers: int, n_kv_heads: int, head_dim: int, seq_len: int,
                   batch: int, dtype_bytes: int, v_head_dim: Optional[int] = None) -> int:
    """Bytes of K and V for every attention layer: one K (head_dim wide) and one V
    (v_head_dim wide, = head_dim unless given) per KV head, token, layer and sequence."""
    dv = head_dim if v_head_dim is None else v_head_dim
    return batch * seq_len * n_attn_layers * n_kv_heads * (head_dim + dv) * dtype_bytes


def ssm_state_bytes(n_layers: int, channels: int, d_state: int, batch: int, dtype_bytes: int) -> int:
    """Bytes of the fixed SSM state: d_state values per channel, layer and sequence."""
    return n_layers * channels * d_state * batch * dtype_bytes


def layer_cache_bytes(cfg, batch: int, max_T: int) -> int:
    """Decode cache of one layer for sequences of up to max_T positions, meta rows
    included: for a producer, KV slots (the meta slots + a ring of `window` slots, or
    one slot per position for a global layer) of 2-byte elements for a bf16 layer (4
    for fp32); then the fp32 SSM state, fp32 conv state and the int32 lengths."""
    esz = 2 if cfg.dtype == 1 else 4
    cap = cfg.n_meta + cfg.window if cfg.window > 0 else max_T
    kv = batch * cfg.n_kv_heads * cap * (cfg.head_dim + cfg.v_head_dim) * esz if cfg.is_kv_producer else 0
    return (kv + ssm_state_bytes(1, cfg.d_inner, cfg.d_state, batch, 4)
            + batch * cfg.d_inner * cfg.d_conv * 4 + batch * 4)
