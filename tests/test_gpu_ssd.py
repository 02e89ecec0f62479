"""GPU parity of the SSD form of the Mamba heads (cfg.ssm_heads > 0: scalar A and Delta per
SSM head, "Lecture 04 - Beyond the Dense Transformer", section 3) against the fp64 oracle,
through the C ABI: the fp32 layer (the sequential scan with per-head values, <= 1e-4),
the bf16 layers (the chunked tensor-core kernel: 64-row chunks, ragged last chunks,
sequences shorter than a chunk and than the conv), the Hymba-1.5B shape with 50 heads,
and decode after prefill through a KV-sharing pair."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import assert_close, to_np, torch_cuda
from test_gpu_decode import _oracle_pair, _Pair
from test_gpu_prefill import _run_prefill, _ws_view

pytestmark = pytest.mark.gpu


def _small_bf16(**kw):
    base = synth.hymba15_layer_cfg(window=40).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                    dt_rank=24, n_meta=8, ssm_heads=10)
    return base.with_(**kw)


def _check_ssd_stages(cfg, r, ref, B, Tp):
    """Delta per head (the GEMM's [rows, ssm_heads] output) and the gated SSM output."""
    import torch
    from hybrid_head_ssm_b200 import runtime as rt
    lay, ws = r["lay"], r["ws"]
    nh, di = cfg.ssm_heads, cfg.d_inner
    P = di // nh
    delta = to_np(_ws_view(ws, lay["delta"], (B, Tp, nh), torch.float32))
    assert_close(delta, ref["delta"][:, :, ::P], cfg, "Delta per head", max_abs=1e-4 if cfg.dtype == 0 else 6e-2)
    mdt = rt.mid_dtype(cfg)
    ypre = to_np(_ws_view(ws, lay["ypre"], (B, Tp, di), mdt))
    Pm = to_np(_ws_view(ws, lay["P"], (B, Tp, lay["ldP"]), mdt))
    zc = cfg.n_q_heads * cfg.head_dim + (cfg.n_kv_heads * (cfg.head_dim + cfg.v_head_dim) if cfg.is_kv_producer else 0) + di
    z = Pm[:, :, zc:zc + di]
    assert_close(ypre * oracle.silu(z), ref["y_ssm"], cfg, "gated SSM output",
                 max_abs=1e-4 if cfg.dtype == 0 else 2.5e-1, rel_l2=5e-3)


def test_tiny_f32_ssd_layer():
    """fp32, 4 heads of 128 channels, B=2, T=77 (ragged scan chunks), perturbed weights."""
    cfg = synth.tiny_layer_cfg().with_(ssm_heads=4, window=16)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 201), cfg, 201)
    x = synth.layer_input(cfg, 2, 77, 202)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    _check_ssd_stages(cfg, r, ref, 2, cfg.n_meta + 77)
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state")
    assert_close(to_np(r["st"].conv), ref["conv"], cfg, "conv state", max_abs=1e-5)


@pytest.mark.parametrize("B,T", [(2, 133), (3, 1), (5, 56), (1, 192)])
def test_bf16_small_ssd_layer(B, T):
    """bf16, 10 heads of 64 channels, perturbed weights. T' = 8 + T rows: 141 (two full
    chunks and a ragged one), 9 (one short chunk), 64 (exactly one), 200."""
    cfg = _small_bf16()
    w = synth.perturbed_weights(synth.layer_weights(cfg, 211), cfg, 211)
    x = synth.layer_input(cfg, B, T, 212)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    mx, rl = assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    print(f"bf16 SSD B={B} T={T}: max abs {mx:.3e}, rel L2 {rl:.3e}")
    _check_ssd_stages(cfg, r, ref, B, cfg.n_meta + T)
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state", max_abs=5e-2)
    assert_close(to_np(r["st"].conv), ref["conv"], cfg, "conv state", max_abs=2e-2)


def test_bf16_ssd_no_meta_shorter_than_the_conv():
    """No meta tokens and T = 2 rows: the conv history is all zeros."""
    cfg = _small_bf16(n_meta=0, window=16)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 221), cfg, 221)
    x = synth.layer_input(cfg, 4, 2, 222)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state", max_abs=5e-2)
    assert_close(to_np(r["st"].conv), ref["conv"], cfg, "conv state", max_abs=2e-2)


def test_bf16_hymba15_ssd_layer():
    """The Hymba-1.5B SWA layer shape with 50 SSM heads of 64 channels, B=1, T=2048."""
    wl = synth.workload("hymba15_swa1024_b1_t2048")
    cfg = wl["cfg"].with_(ssm_heads=50)
    w = synth.layer_weights(cfg, 231)
    x = synth.layer_input(cfg, 1, 2048, 232)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    mx, rl = assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    print(f"hymba15 SSD layer: max abs {mx:.3e}, rel L2 {rl:.3e}")
    _check_ssd_stages(cfg, r, ref, 1, cfg.n_meta + 2048)
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state", max_abs=5e-2)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ssd_pair_decode_matches_oracle(dtype):
    """Prefill, then decode steps through a KV-sharing pair of SSD layers (ring wraps)."""
    if dtype == "f32":
        base = synth.tiny_layer_cfg().with_(window=8, ssm_heads=8)
        B, T0, steps, seed = 2, 10, 12, 241
    else:
        base = _small_bf16(window=24)
        B, T0, steps, seed = 3, 70, 10, 242
    ca, cb = base, base.with_(is_kv_producer=0)
    wa, wb = synth.layer_weights(ca, seed), synth.layer_weights(cb, seed + 1)
    if dtype == "f32":
        wa, wb = synth.perturbed_weights(wa, ca, seed), synth.perturbed_weights(wb, cb, seed + 1)
    x = synth.layer_input(ca, B, T0 + steps, seed + 2)
    cap = ca.n_meta + ca.window
    g = _Pair(ca, cb, wa, wb, B, T0, cap)
    g.prefill(x[:, :T0])
    o = _oracle_pair(ca, cb, wa, wb, x[:, :T0], cap)
    for t in range(T0, T0 + steps):
        ya, yb = g.step(x[:, t])
        ra = oracle.mixer_decode(ca, wa, x[:, t], o["cache"], o["ha"], o["ca"], residual=True)
        rb = oracle.mixer_decode(cb, wb, ra, o["cache"], o["hb"], o["cb"], residual=True)
        assert_close(to_np(ya), ra, ca, f"producer step {t}")
        assert_close(to_np(yb), rb, cb, f"consumer step {t}")
    assert_close(to_np(g.sa.h), o["ha"], ca, "producer state after decode", max_abs=1e-4 if dtype == "f32" else 5e-2)
    assert g.hy.hymba_get_device_status(None) == 0
