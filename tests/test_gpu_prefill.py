"""GPU parity of hymba_mixer_prefill against the fp64 CPU oracle, element by element,
through the C ABI. Stage outputs left in the workspace (projection, Delta, attention
output, y_pre, fused U) are compared too, so a failure names the stage."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import assert_close, errors, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _run_prefill(cfg, w, x, *, kv_from=None, cache_cap=0, flags=0, state=True):
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    B, T = x.shape[0], (x.shape[1] - cfg.n_meta if flags & hy.HYMBA_X_HAS_META else x.shape[1])
    Tp = cfg.n_meta + T
    layer = rt.DeviceLayer(cfg, w)
    xd = rt.to_device(x, cfg)
    yd = torch.empty((B, Tp, cfg.d_model), dtype=rt.act_dtype(cfg), device="cuda")
    if kv_from is None:
        kv = rt.KV(cfg, B, seq_cap=Tp, cache_cap=cache_cap)
        kvs = kv.s
    else:
        kv = kv_from
        kvs = hy.hymba_kv()
        hy.check(hy.hymba_kv_share(ctypes.byref(kv_from.s), ctypes.byref(layer.c), ctypes.byref(kvs)))
    st = rt.State(cfg, B) if state else None
    ws = rt.workspace(cfg, B, T, hy.HYMBA_MODE_PREFILL)
    ws.fill_(0xFF)  # garbage: every stage must write what it later reads
    rt.prefill(layer, xd, T, kv, yd, ws, st, flags, kv_struct_override=kvs)
    torch.cuda.synchronize()
    status = hy.hymba_get_device_status(None)
    assert status == 0, (status, hy.device_diag())
    lay = hy.workspace_layout(layer.c, B, T, hy.HYMBA_MODE_PREFILL)
    return dict(y=yd, kv=kv, st=st, ws=ws, lay=lay, layer=layer)


def _ws_view(ws, off, shape, dtype):
    import torch
    n = int(np.prod(shape))
    esz = torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + n * esz].view(dtype).view(*shape)


def _check_stages(cfg, r, ref, B, Tp, delta_written=True):
    import torch
    from hybrid_head_ssm_b200 import runtime as rt
    lay, ws = r["lay"], r["ws"]
    mdt = rt.mid_dtype(cfg)
    di, H, dv = cfg.d_inner, cfg.n_q_heads, cfg.v_head_dim
    # a wide bf16 batch computes Delta inside the scan kernel (no Delta tensor)
    delta = to_np(_ws_view(ws, lay["delta"], (B, Tp, di), torch.float32)) if delta_written else None
    o = to_np(_ws_view(ws, lay["O"], (B, Tp, H * dv), mdt))
    u = to_np(_ws_view(ws, lay["U"], (B, Tp, di), rt.act_dtype(cfg)))
    ypre = to_np(_ws_view(ws, lay["ypre"], (B, Tp, di), mdt))
    P = to_np(_ws_view(ws, lay["P"], (B, Tp, lay["ldP"]), mdt))
    zc = cfg.n_q_heads * cfg.head_dim + (cfg.n_kv_heads * (cfg.head_dim + cfg.v_head_dim) if cfg.is_kv_producer else 0) + di
    z = P[:, :, zc:zc + di]
    tol = dict(max_abs=1e-4 if cfg.dtype == 0 else 6e-2, rel_l2=5e-3)
    if delta is not None:
        assert_close(delta, ref["delta"], cfg, "Delta", max_abs=tol["max_abs"])
    assert_close(ypre * oracle.silu(z), ref["y_ssm"], cfg, "gated SSM output", max_abs=1e-4 if cfg.dtype == 0 else 2.5e-1,
                 rel_l2=5e-3)
    assert_close(o, ref["o_attn"], cfg, "attention output", **tol)
    assert_close(u, ref["u"], cfg, "fused U", max_abs=1e-4 if cfg.dtype == 0 else 1.5e-1, rel_l2=5e-3)


@pytest.mark.parametrize("perturb", [False, True])
def test_tiny_f32_layer(perturb):
    """Tiny fp32 layer (B=1, T=256 + 16 meta, window 64): y and every stage <= 1e-4."""
    wl = synth.workload("tiny_f32_b1_t256")
    cfg = wl["cfg"]
    w = synth.layer_weights(cfg, wl["seed"])
    if perturb:
        w = synth.perturbed_weights(w, cfg, 5)
    x = synth.layer_input(cfg, wl["B"], wl["T"], wl["seed"])
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    B, Tp = wl["B"], cfg.n_meta + wl["T"]
    assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    _check_stages(cfg, r, ref, B, Tp)
    assert_close(to_np(r["kv"].k_seq), ref["k"], cfg, "K after RoPE")
    assert_close(to_np(r["kv"].v_seq), ref["v"], cfg, "V")
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state")
    assert_close(to_np(r["st"].conv), ref["conv"], cfg, "conv state", max_abs=1e-5)


def test_tiny_f32_ragged_batch_and_tails():
    """B=3, T=77 (not a multiple of any tile), window 5, n_meta 16: ragged tails
    in the GEMM, attention and scan tiles."""
    cfg = synth.tiny_layer_cfg().with_(window=5)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 8), cfg, 8)
    x = synth.layer_input(cfg, 3, 77, 8)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state")


def test_tiny_f32_global_and_no_meta():
    """Global attention (window 0) and a layer without meta tokens."""
    for kw in (dict(window=0), dict(n_meta=0, window=16)):
        cfg = synth.tiny_layer_cfg().with_(**kw)
        w = synth.layer_weights(cfg, 9)
        x = synth.layer_input(cfg, 2, 50, 9)
        ref = oracle.mixer_prefill(cfg, w, x)
        r = _run_prefill(cfg, w, x)
        assert_close(to_np(r["y"]), ref["y"], cfg, f"y {kw}")


def test_tiny_f32_kv_share_and_residual_stack():
    """Producer then consumer (hymba_kv_share, no K/V rows of its own), residual
    stack with the consumer's input = the producer's output rows (meta included)."""
    base = synth.tiny_layer_cfg().with_(window=12)
    ca, cb = base, base.with_(is_kv_producer=0)
    wa = synth.perturbed_weights(synth.layer_weights(ca, 21), ca, 21)
    wb = synth.perturbed_weights(synth.layer_weights(cb, 22), cb, 22)
    x = synth.layer_input(ca, 2, 40, 23)
    ra = oracle.mixer_prefill(ca, wa, x, residual=True)
    rb = oracle.mixer_prefill(cb, wb, ra["y"], kv_shared=(ra["k"], ra["v"]), residual=True, x_has_meta=True)
    import hybrid_head_ssm_b200 as hy
    ga = _run_prefill(ca, wa, x, flags=hy.HYMBA_ADD_RESIDUAL)
    assert_close(to_np(ga["y"]), ra["y"], ca, "producer y")
    # the consumer reads the GPU producer's K/V; its input is the GPU producer's output
    from hybrid_head_ssm_b200 import runtime as rt
    torch = torch_cuda()
    lb = rt.DeviceLayer(cb, wb)
    kvs = hy.hymba_kv()
    hy.check(hy.hymba_kv_share(ctypes.byref(ga["kv"].s), ctypes.byref(lb.c), ctypes.byref(kvs)))
    yb = ga["y"].clone()
    ws = rt.workspace(cb, 2, 40, hy.HYMBA_MODE_PREFILL)
    rt.prefill(lb, yb, 40, ga["kv"], yb, ws, None, hy.HYMBA_X_HAS_META | hy.HYMBA_ADD_RESIDUAL,
               kv_struct_override=kvs)  # in place: y == x
    torch.cuda.synchronize()
    assert_close(to_np(yb), rb["y"], cb, "consumer y (in place)")


def test_bf16_hymba15_swa_layer():
    """Hymba-1.5B-shaped SWA layer, bf16, B=1, T=2048 + 128 meta: the full output."""
    wl = synth.workload("hymba15_swa1024_b1_t2048")
    cfg = wl["cfg"]
    w = synth.layer_weights(cfg, wl["seed"])
    x = synth.layer_input(cfg, wl["B"], wl["T"], wl["seed"])
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    mx, rl = assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    print(f"hymba15 swa layer: max abs {mx:.3e}, rel L2 {rl:.3e}")
    _check_stages(cfg, r, ref, wl["B"], cfg.n_meta + wl["T"])
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state", max_abs=5e-2)


def test_bf16_small_perturbed_layer():
    """A small bf16 layer with every per-channel parameter away from its default,
    ragged T, KV share to a consumer."""
    cfg = synth.hymba15_layer_cfg(window=40).with_(d_model=256, n_q_heads=5, n_kv_heads=1,
                                                   d_inner=640, dt_rank=24, n_meta=8)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 31), cfg, 31)
    x = synth.layer_input(cfg, 2, 133, 31)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    assert_close(to_np(r["y"]), ref["y"], cfg, "y")
    cc = cfg.with_(is_kv_producer=0)
    wc = synth.perturbed_weights(synth.layer_weights(cc, 32), cc, 32)
    refc = oracle.mixer_prefill(cc, wc, x, kv_shared=(ref["k"], ref["v"]))
    rc = _run_prefill(cc, wc, x, kv_from=r["kv"])
    assert_close(to_np(rc["y"]), refc["y"], cc, "consumer y")


def test_bf16_global_layer_b4_t8192_sampled_rows():
    """Global layer, B=4, T=8192 + 128 meta, run in full on the GPU; the oracle
    recomputes sequences 0 and 3 (rows are independent)."""
    wl = synth.workload("hymba15_global_b4_t8192")
    cfg = wl["cfg"]
    w = synth.layer_weights(cfg, wl["seed"])
    x = synth.layer_input(cfg, wl["B"], wl["T"], wl["seed"])
    r = _run_prefill(cfg, w, x)
    y = to_np(r["y"])
    for b in (0, 3):
        ref = oracle.mixer_prefill_row(cfg, w, x[b])
        mx, rl = assert_close(y[b], ref["y"], cfg, f"y row {b}")
        print(f"global layer row {b}: max abs {mx:.3e}, rel L2 {rl:.3e}")


def test_prefill_fills_decode_ring_bit_exact():
    """A producer's prefill with a ring smaller than the sequence copies the meta
    rows and the newest positions into slot n_meta + (p - n_meta) mod R: compare
    the cache with the prefill's own K/V rows, bit for bit."""
    torch = torch_cuda()
    cfg = synth.tiny_layer_cfg().with_(window=8)
    w = synth.layer_weights(cfg, 3)
    x = synth.layer_input(cfg, 2, 37, 3)
    cap = cfg.n_meta + 8
    r = _run_prefill(cfg, w, x, cache_cap=cap)
    kv = r["kv"]
    Tp = cfg.n_meta + 37
    ks, vs = kv.k_seq.cpu(), kv.v_seq.cpu()
    kc, vc = kv.k_cache.cpu(), kv.v_cache.cpu()
    for p in list(range(cfg.n_meta)) + list(range(Tp - 8, Tp)):
        s = oracle.ring_slot(p, cfg.n_meta, 8)
        assert torch.equal(kc[:, :, s], ks[:, :, p]) and torch.equal(vc[:, :, s], vs[:, :, p]), p
    assert kv.len.cpu().tolist() == [Tp, Tp]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_consumer_with_affine_shared_kv(dtype):
    """A consumer that adapts the shared K and V ("Hymba Guide", Cross-Layer KV Cache
    Sharing: K~ = K * w_scale + b_bias per KV head, V likewise) reads the GPU producer's
    K/V; its output and attention stage match the oracle's literal adaptation."""
    if dtype == "f32":
        base = synth.tiny_layer_cfg().with_(window=24)
        B, T = 2, 90
    else:
        base = synth.hymba15_layer_cfg(window=40).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                        dt_rank=24, n_meta=8)
        B, T = 2, 133
    cp, cc = base, base.with_(is_kv_producer=0)
    wp = synth.layer_weights(cp, 41)
    wc = dict(synth.perturbed_weights(synth.layer_weights(cc, 42), cc, 42), **synth.affine_kv(cc, 43))
    x = synth.layer_input(cp, B, T, 44)
    refp = oracle.mixer_prefill(cp, wp, x)
    refc = oracle.mixer_prefill(cc, wc, x, kv_shared=(refp["k"], refp["v"]))
    rp = _run_prefill(cp, wp, x)
    rc = _run_prefill(cc, wc, x, kv_from=rp["kv"])
    mx, rl = assert_close(to_np(rc["y"]), refc["y"], cc, "consumer y with adapted K/V")
    print(f"affine shared KV consumer ({dtype}): max abs {mx:.3e}, rel L2 {rl:.3e}")
    import torch
    from hybrid_head_ssm_b200 import runtime as rt
    lay = rc["lay"]
    o = to_np(_ws_view(rc["ws"], lay["O"], (B, cc.n_meta + T, cc.n_q_heads * cc.v_head_dim), rt.mid_dtype(cc)))
    # the workspace holds the attention before the V adaptation (applied in the fusion)
    nk, rep = cc.n_kv_heads * cc.head_dim, cc.n_q_heads // cc.n_kv_heads
    vs = np.repeat(wc["kv_scale"][nk:].reshape(cc.n_kv_heads, cc.v_head_dim), rep, axis=0).ravel()
    vb = np.repeat(wc["kv_bias"][nk:].reshape(cc.n_kv_heads, cc.v_head_dim), rep, axis=0).ravel()
    o_ref = (refc["o_attn"] - vb) / vs  # per query head h, the V adaptation of its KV head
    assert_close(o, o_ref, cc, "attention output (before the V adaptation)",
                 max_abs=1e-4 if cc.dtype == 0 else 2e-2)
    with pytest.raises(Exception):
        # a producer may not carry the adaptation
        _run_prefill(cp, dict(wp, **synth.affine_kv(cp, 45)), x)


@pytest.mark.parametrize("case", ["f32_tiny", "bf16_small", "bf16_hymba15"])
def test_concat_fusion_layer(case):
    """The concat fusion ("Hymba Guide", Parallel Hybrid-Head Layer Formulation:
    y = W_o(Concat[MambaHeads(x), AttentionHeads(x)])) with V head dim 64 = the Q/K
    head dim: attention output H * 64 wide, U = [Mamba | attention], W_o over both."""
    if case == "f32_tiny":
        cfg = synth.tiny_layer_cfg().with_(fusion=1, v_head_dim=64, window=24)
        B, T = 2, 90
    elif case == "bf16_small":
        cfg = synth.hymba15_layer_cfg(window=40).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                       dt_rank=24, n_meta=8, fusion=1, v_head_dim=64)
        B, T = 2, 133
    else:
        cfg = synth.hymba15_layer_cfg(window=1024).with_(fusion=1, v_head_dim=64)
        B, T = 1, 1500
    w = synth.perturbed_weights(synth.layer_weights(cfg, 111), cfg, 111)
    x = synth.layer_input(cfg, B, T, 112)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    mx, rl = assert_close(to_np(r["y"]), ref["y"], cfg, "y (concat fusion)")
    print(f"concat fusion {case}: max abs {mx:.3e}, rel L2 {rl:.3e}")
    from hybrid_head_ssm_b200 import runtime as rt
    lay = r["lay"]
    Tp = cfg.n_meta + T
    o = to_np(_ws_view(r["ws"], lay["O"], (B, Tp, cfg.n_q_heads * cfg.v_head_dim), rt.mid_dtype(cfg)))
    assert_close(o, ref["o_attn"], cfg, "attention output (dv 64)", max_abs=1e-4 if cfg.dtype == 0 else 2e-2)
    # a consumer of the concat producer's 64-wide V
    cc = cfg.with_(is_kv_producer=0)
    wc = synth.perturbed_weights(synth.layer_weights(cc, 113), cc, 113)
    refc = oracle.mixer_prefill(cc, wc, x, kv_shared=(ref["k"], ref["v"]))
    rc = _run_prefill(cc, wc, x, kv_from=r["kv"])
    assert_close(to_np(rc["y"]), refc["y"], cc, "consumer y (concat fusion)")


@pytest.mark.parametrize("T", [70, 10, 24])
def test_bf16_many_sequences_use_the_wide_scan(T):
    """A batch wide enough (B * d_inner / 64 >= 2 * SMs) for the wide scan (two threads
    per channel, Delta computed inside it): 30 sequences of a small bf16 layer with 8 meta
    rows + T: a ragged last chunk (78 rows), one short chunk (18), exactly one chunk (32);
    y, the final SSM state and the conv state."""
    cfg = synth.hymba15_layer_cfg(window=24).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                   dt_rank=24, n_meta=8)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 141), cfg, 141)
    B = 30
    x = synth.layer_input(cfg, B, T, 142)
    ref = oracle.mixer_prefill(cfg, w, x)
    r = _run_prefill(cfg, w, x)
    mx, rl = assert_close(to_np(r["y"]), ref["y"], cfg, "y (wide scan)")
    print(f"wide scan batch: max abs {mx:.3e}, rel L2 {rl:.3e}")
    _check_stages(cfg, r, ref, B, cfg.n_meta + T, delta_written=False)
    assert_close(to_np(r["st"].h), ref["h"], cfg, "final SSM state", max_abs=5e-2)
    assert_close(to_np(r["st"].conv), ref["conv"], cfg, "conv state", max_abs=2e-2)
