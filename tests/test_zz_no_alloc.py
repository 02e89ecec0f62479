"""hymba_attn_decode_static: the decode attention for callers that cannot allocate
device memory (no workspace argument; its scratch is a fixed device array inside the
library). Checked against the attention of hymba_mixer_decode for the same query and
cache: the mixer leaves its split-KV partials in its workspace, merged here on the host
by the softmax rescaling rule, on two calls in a row (the second call reuses the array
the first one left behind).

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest

import synth
from gpu_helpers import BF16_MAX_ABS, BF16_REL_L2, errors, merge_split_partials, torch_cuda

pytestmark = pytest.mark.gpu


def _decoded_layer(cfg, B, T0, cache_cap, seed):
    """One producer layer prefilled with T0 tokens, then one hymba_mixer_decode step;
    returns the pieces the static call needs and the mixer's own attention output."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    w = synth.layer_weights(cfg, seed)
    layer = rt.DeviceLayer(cfg, w)
    kv = rt.KV(cfg, B, seq_cap=cfg.n_meta + T0, cache_cap=cache_cap)
    st = rt.State(cfg, B)
    x = synth.layer_input(cfg, B, T0 + 1, seed)
    y0 = torch.empty((B, cfg.n_meta + T0, cfg.d_model), dtype=rt.act_dtype(cfg), device="cuda")
    rt.prefill(layer, rt.to_device(x[:, :T0], cfg), T0, kv, y0, rt.workspace(cfg, B, T0, hy.HYMBA_MODE_PREFILL), st)
    ws = rt.workspace(cfg, B, cache_cap, hy.HYMBA_MODE_DECODE)
    xt = rt.to_device(x[:, T0], cfg)
    yt = torch.empty_like(xt)
    rt.decode(layer, xt, kv.s, st, yt, ws)
    torch.cuda.synchronize()
    lay = hy.workspace_layout(layer.c, B, cache_cap, hy.HYMBA_MODE_DECODE)
    mdt = rt.mid_dtype(cfg)
    esz = torch.tensor([], dtype=mdt).element_size()
    H, dh, dv = cfg.n_q_heads, cfg.head_dim, cfg.v_head_dim
    ldp = lay["ldP"]
    # the query rows (after RoPE) sit in the projection block of the workspace
    q = ws[lay["P"]:lay["P"] + B * ldp * esz].view(mdt).view(B, ldp)
    ns = lay["n_split"]
    # records of dv + 4 floats: dv sums, the max logit, the sum of p, two pad words
    n_part = B * H * ns * (dv + 4)
    part = ws[lay["part"]:lay["part"] + n_part * 4].view(torch.float32).view(B, H, ns, dv + 4)
    o_ref = merge_split_partials(part[..., :dv + 2].double().cpu().numpy()).reshape(B, H * dv)
    return dict(layer=layer, kv=kv, q=q, ldp=ldp, o_ref=o_ref, mdt=mdt)


@pytest.mark.parametrize("kind", ["bf16_hymba15_ring", "f32_tiny_global", "bf16_hymba15_wrapped_5splits",
                                  "f32_tiny_global_3splits"])
def test_static_decode_attention_matches_mixer_decode(kind):
    """One split (80-slot caches) and several: the 1.5B ring of 1024 + 128 meta slots
    after 1500 prompt tokens (wrapped; 5 splits of 256 keys here, 9 of 128 in the
    mixer) and a global fp32 cache of 616 slots (3 splits)."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    if kind == "bf16_hymba15_ring":
        cfg = synth.hymba15_layer_cfg(window=64).with_(n_meta=16)
        B, T0, cap = 16, 150, 16 + 64
    elif kind == "f32_tiny_global":
        cfg = synth.tiny_layer_cfg().with_(window=0)
        B, T0, cap = 3, 40, 16 + 64
    elif kind == "bf16_hymba15_wrapped_5splits":
        cfg = synth.hymba15_layer_cfg(window=1024)
        B, T0, cap = 8, 1500, 128 + 1024
    else:
        cfg = synth.tiny_layer_cfg().with_(window=0)
        B, T0, cap = 2, 520, 16 + 600
    r = _decoded_layer(cfg, B, T0, cap, seed=5)
    H, dv = cfg.n_q_heads, cfg.v_head_dim
    for call in range(2):
        o = torch.full((B, H * dv), float("nan"), dtype=r["mdt"], device="cuda")
        rc = hy.hymba_attn_decode_static(ctypes.byref(r["layer"].c), r["q"].data_ptr(), r["ldp"],
                                         ctypes.byref(r["kv"].s), o.data_ptr(), B, hy.current_stream_ptr())
        assert rc == hy.HYMBA_OK, hy.hymba_strerror(rc)
        torch.cuda.synchronize()
        assert hy.hymba_get_device_status(None) == hy.HYMBA_OK
        got = o.float().cpu().numpy()
        mx, rl = errors(got, r["o_ref"])
        if cfg.dtype == 1:
            assert mx <= BF16_MAX_ABS and rl <= BF16_REL_L2, (call, mx, rl)
        else:
            assert mx <= 1e-4, (call, mx)


def test_static_decode_attention_rejects_requests_beyond_its_scratch():
    """B * n_q_heads * splits * (v_head_dim + 4) * 4 bytes must fit the fixed 8 MiB."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    cfg = synth.hymba15_layer_cfg(window=0)
    B, cap = 64, 128 + 8192  # 33 splits: 64 * 25 * 33 * 132 * 4 bytes > 8 MiB
    kv = hy.kv_struct(cfg, B)
    kv.k_cache = kv.v_cache = kv.len = 1 << 30  # never dereferenced: the check comes first
    kv.cache_cap = cap
    rc = hy.hymba_attn_decode_static(ctypes.byref(hy.cfg_struct(cfg)), 1 << 30, cfg.n_q_heads * 64,
                                     ctypes.byref(kv), 1 << 30, B, None)
    assert rc == hy.HYMBA_ERR_SCRATCH_LIMIT
    assert "scratch" in hy.hymba_strerror(rc).decode()


def test_static_decode_attention_visible_set_bit_exact():
    """The allocation-free entry point attends to exactly the visible cache slots
    (K = 0, one-hot V; see test_gpu_visibility): the 1.5B ring of 1024 + 128 slots
    before and after it wraps (5 splits of 256 keys), and a short window."""
    from test_gpu_visibility import _decode_visibility
    cfg = synth.hymba15_layer_cfg(1024)
    _decode_visibility(cfg, 8, 128 + 1024, (1, 300, 128 + 1024, 128 + 4096 + 1), 31, static=True)
    small = cfg.with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640, dt_rank=24, n_meta=16, window=7)
    _decode_visibility(small, 3, 16 + 7, (5, 23, 61), 32, static=True)
