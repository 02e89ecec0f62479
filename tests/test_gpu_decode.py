"""GPU parity of hymba_mixer_decode (one new token per sequence, KV ring + O(1) SSM
state) against the fp64 CPU oracle, through the C ABI, and the bit-exact checks
of the ring writes."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import assert_close, to_np, torch_cuda

pytestmark = pytest.mark.gpu


class _Pair:
    """A KV-sharing layer pair on the GPU: producer A, consumer B, residual stack."""

    def __init__(self, ca, cb, wa, wb, B, Tprompt, cache_cap):
        torch = torch_cuda()
        import hybrid_head_ssm_b200 as hy
        from hybrid_head_ssm_b200 import runtime as rt
        self.hy, self.rt, self.torch = hy, rt, torch
        self.ca, self.cb, self.B = ca, cb, B
        self.la, self.lb = rt.DeviceLayer(ca, wa), rt.DeviceLayer(cb, wb)
        Tp = ca.n_meta + Tprompt
        self.kv = rt.KV(ca, B, seq_cap=Tp, cache_cap=cache_cap)
        self.kvb = hy.hymba_kv()
        hy.check(hy.hymba_kv_share(ctypes.byref(self.kv.s), ctypes.byref(self.lb.c), ctypes.byref(self.kvb)))
        self.sa, self.sb = rt.State(ca, B), rt.State(cb, B)
        self.wsa = rt.workspace(ca, B, Tprompt, hy.HYMBA_MODE_PREFILL)
        self.wsb = rt.workspace(cb, B, Tprompt, hy.HYMBA_MODE_PREFILL)
        self.wda = rt.workspace(ca, B, cache_cap, hy.HYMBA_MODE_DECODE)
        self.wdb = rt.workspace(cb, B, cache_cap, hy.HYMBA_MODE_DECODE)
        self.Tprompt = Tprompt
        # residual stream between the two layers: fp32 for bf16 layers
        self.flags = rt.stream_flags(ca)
        self.io_f32 = bool(self.flags & hy.HYMBA_IO_F32) or ca.dtype == 0

    def prefill(self, x):
        hy, rt, torch = self.hy, self.rt, self.torch
        xd = rt.to_device(x, self.ca, io_f32=self.io_f32)
        ya = torch.empty((self.B, self.ca.n_meta + self.Tprompt, self.ca.d_model), dtype=xd.dtype, device="cuda")
        rt.prefill(self.la, xd, self.Tprompt, self.kv, ya, self.wsa, self.sa, self.flags)
        yb = torch.empty_like(ya)
        rt.prefill(self.lb, ya, self.Tprompt, self.kv, yb, self.wsb, self.sb,
                   hy.HYMBA_X_HAS_META | self.flags, kv_struct_override=self.kvb)
        return ya, yb

    def step(self, x_t):
        hy, rt, torch = self.hy, self.rt, self.torch
        xd = rt.to_device(x_t, self.ca, io_f32=self.io_f32)
        ya = torch.empty_like(xd)
        yb = torch.empty_like(xd)
        rt.decode(self.la, xd, self.kv.s, self.sa, ya, self.wda, self.flags)
        rt.decode(self.lb, ya, self.kvb, self.sb, yb, self.wdb, self.flags)
        return ya, yb


def _oracle_pair(ca, cb, wa, wb, x_prompt, cache_cap):
    pa = oracle.mixer_prefill(ca, wa, x_prompt, residual=True)
    pb = oracle.mixer_prefill(cb, wb, pa["y"], kv_shared=(pa["k"], pa["v"]), residual=True, x_has_meta=True)
    cache = oracle.cache_from_prefill(ca, pa["k"], pa["v"], cache_cap)
    return dict(cache=cache, ha=pa["h"].copy(), ca=pa["conv"].copy(), hb=pb["h"].copy(),
                cb=pb["conv"].copy(), ya=pa["y"], yb=pb["y"])


@pytest.mark.parametrize("window", [8, 0])
def test_tiny_f32_pair_decode_matches_oracle(window):
    """Prefill 10 tokens, then decode 14 through a producer/consumer pair; window 8
    uses an 8-slot ring that wraps; window 0 (global) a cache holding all positions."""
    base = synth.tiny_layer_cfg().with_(window=window)
    ca, cb = base, base.with_(is_kv_producer=0)
    wa = synth.perturbed_weights(synth.layer_weights(ca, 61), ca, 61)
    wb = synth.perturbed_weights(synth.layer_weights(cb, 62), cb, 62)
    B, T0, steps = 3, 10, 14
    x = synth.layer_input(ca, B, T0 + steps, 63)
    cap = ca.n_meta + (window if window > 0 else T0 + steps)
    g = _Pair(ca, cb, wa, wb, B, T0, cap)
    ga, gb = g.prefill(x[:, :T0])
    o = _oracle_pair(ca, cb, wa, wb, x[:, :T0], cap)
    assert_close(to_np(gb), o["yb"], cb, "prefill y of the consumer")
    for t in range(T0, T0 + steps):
        ya, yb = g.step(x[:, t])
        ra = oracle.mixer_decode(ca, wa, x[:, t], o["cache"], o["ha"], o["ca"], residual=True)
        rb = oracle.mixer_decode(cb, wb, ra, o["cache"], o["hb"], o["cb"], residual=True)
        assert_close(to_np(ya), ra, ca, f"producer step {t}")
        assert_close(to_np(yb), rb, cb, f"consumer step {t}")
    assert g.kv.len.cpu().tolist() == [ca.n_meta + T0 + steps] * B
    assert_close(to_np(g.sa.h), o["ha"], ca, "producer state")
    assert_close(to_np(g.sb.conv), o["cb"], cb, "consumer conv state")
    assert g.hy.hymba_get_device_status(None) == 0


@pytest.mark.parametrize("dt_rank", [24, 130, 264])
def test_bf16_small_pair_decode_matches_oracle(dt_rank):
    """The decode SSM step stages W_dt with wide loads for an even dt_rank <= 128 (24)
    and with its general loop otherwise: one pass (130) or two (264)."""
    base = synth.hymba15_layer_cfg(window=24).with_(d_model=256, n_q_heads=5, n_kv_heads=1,
                                                    d_inner=640, dt_rank=dt_rank, n_meta=8)
    ca, cb = base, base.with_(is_kv_producer=0)
    wa = synth.layer_weights(ca, 71)
    wb = synth.layer_weights(cb, 72)
    B, T0, steps = 4, 40, 12
    x = synth.layer_input(ca, B, T0 + steps, 73)
    cap = ca.n_meta + 24
    g = _Pair(ca, cb, wa, wb, B, T0, cap)
    g.prefill(x[:, :T0])
    o = _oracle_pair(ca, cb, wa, wb, x[:, :T0], cap)
    for t in range(T0, T0 + steps):
        ya, yb = g.step(x[:, t])
        ra = oracle.mixer_decode(ca, wa, x[:, t], o["cache"], o["ha"], o["ca"], residual=True)
        rb = oracle.mixer_decode(cb, wb, ra, o["cache"], o["hb"], o["cb"], residual=True)
        assert_close(to_np(ya), ra, ca, f"producer step {t}")
        assert_close(to_np(yb), rb, cb, f"consumer step {t}")


def test_decode_ring_writes_bit_exact():
    """With one-hot inputs, the new V row of a producer is exactly a column of W_V:
    after each decode step exactly the ring slot n_meta + (p - n_meta) mod R holds it,
    and every other slot is unchanged."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    cfg = synth.tiny_layer_cfg().with_(window=6)
    w = synth.layer_weights(cfg, 81)
    B, T0, R = 2, 9, 6
    cap = cfg.n_meta + R
    layer = rt.DeviceLayer(cfg, w)
    kv = rt.KV(cfg, B, seq_cap=cfg.n_meta + T0, cache_cap=cap)
    st = rt.State(cfg, B)
    x0 = rt.to_device(synth.layer_input(cfg, B, T0, 82), cfg)
    y0 = torch.empty((B, cfg.n_meta + T0, cfg.d_model), device="cuda")
    rt.prefill(layer, x0, T0, kv, y0, rt.workspace(cfg, B, T0, hy.HYMBA_MODE_PREFILL), st)
    wsd = rt.workspace(cfg, B, cap, hy.HYMBA_MODE_DECODE)
    H, G, dh, dv = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim
    v_rows = w["w_in"][H * dh + G * dh: H * dh + G * dh + G * dv]  # [G*dv, d]
    for step in range(15):
        before = kv.v_cache.clone()
        p = cfg.n_meta + T0 + step
        col = (5 * step + 1) % cfg.d_model
        xt = torch.zeros((B, cfg.d_model), device="cuda")
        xt[:, col] = 1.0
        yt = torch.empty_like(xt)
        rt.decode(layer, xt, kv.s, st, yt, wsd)
        torch.cuda.synchronize()
        slot = oracle.ring_slot(p, cfg.n_meta, R)
        expect = torch.from_numpy(v_rows[:, col].reshape(G, dv).astype(np.float32))
        after = kv.v_cache.cpu()
        for b in range(B):
            assert torch.equal(after[b, :, slot], expect), (step, slot)
        mask = torch.ones(cap, dtype=torch.bool)
        mask[slot] = False
        assert torch.equal(after[:, :, mask], before.cpu()[:, :, mask])
        assert kv.len.cpu().tolist() == [p + 1] * B


def test_decode_span_longer_than_ring_reports_range_error():
    """A global layer whose cache ring is shorter than the history cannot attend to
    every position: the step records HYMBA_ERR_DEVICE_RANGE in the status word (read
    on the host) and writes a zero attention output, with no fault."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    cfg = synth.tiny_layer_cfg().with_(window=0)
    w = synth.layer_weights(cfg, 91)
    B, T0 = 1, 20
    cap = cfg.n_meta + 8
    layer = rt.DeviceLayer(cfg, w)
    kv = rt.KV(cfg, B, seq_cap=cfg.n_meta + T0, cache_cap=cap)
    st = rt.State(cfg, B)
    x0 = rt.to_device(synth.layer_input(cfg, B, T0, 92), cfg)
    y0 = torch.empty((B, cfg.n_meta + T0, cfg.d_model), device="cuda")
    rt.prefill(layer, x0, T0, kv, y0, rt.workspace(cfg, B, T0, hy.HYMBA_MODE_PREFILL), st)
    assert hy.hymba_get_device_status(None) == hy.HYMBA_OK
    xt = rt.to_device(synth.layer_input(cfg, B, 1, 93)[:, 0], cfg)
    yt = torch.empty_like(xt)
    rt.decode(layer, xt, kv.s, st, yt, rt.workspace(cfg, B, cap, hy.HYMBA_MODE_DECODE))
    assert hy.hymba_get_device_status(None) == hy.HYMBA_ERR_DEVICE_RANGE
    assert hy.hymba_get_device_status(None) == hy.HYMBA_OK  # read clears it
    assert torch.isfinite(yt).all()


def test_hymba15_decode_pair_b64_sampled_rows():
    """Decode step of the Hymba-1.5B-shaped pair: B=64 sequences, a 4096-token prompt
    + 128 meta prefilled through both layers into a 1024-slot ring, then one new
    token. The oracle recomputes sequences 0 and 63 (prompt and step) on its own."""
    wl = synth.workload("hymba15_decode_pair_b64_p4096")
    ca = wl["cfg"]
    cb = ca.with_(is_kv_producer=0)
    seed, B, T = wl["seed"], wl["B"], wl["T"]
    wa, wb = synth.layer_weights(ca, seed * 1000), synth.layer_weights(cb, seed * 1000 + 1)
    x = synth.layer_input(ca, B, T, seed)
    xt = synth.layer_input(ca, B, 1, seed, tag=1)[:, 0]
    cap = ca.n_meta + ca.window
    g = _Pair(ca, cb, wa, wb, B, T, cap)
    g.prefill(x)
    ya, yb = g.step(xt)
    ya, yb = to_np(ya), to_np(yb)
    for b in (0, 63):
        o = _oracle_pair(ca, cb, wa, wb, x[b:b + 1], cap)
        ra = oracle.mixer_decode(ca, wa, xt[b:b + 1], o["cache"], o["ha"], o["ca"], residual=True)
        rb = oracle.mixer_decode(cb, wb, ra, o["cache"], o["hb"], o["cb"], residual=True)
        mx, rl = assert_close(ya[b:b + 1], ra, ca, f"producer row {b}")
        mx2, rl2 = assert_close(yb[b:b + 1], rb, cb, f"consumer row {b}")
        print(f"decode pair row {b}: A {mx:.3e}/{rl:.3e}, B {mx2:.3e}/{rl2:.3e}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pair_decode_with_affine_shared_kv(dtype):
    """Decode through a pair whose consumer adapts the shared K/V: the query scale and
    the V transform act in the decode path as in the oracle's literal adaptation of the
    cached K, V (window 8 / 24 rings that wrap)."""
    if dtype == "f32":
        base = synth.tiny_layer_cfg().with_(window=8)
        B, T0, steps, seed = 2, 10, 12, 81
    else:
        base = synth.hymba15_layer_cfg(window=24).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                        dt_rank=24, n_meta=8)
        B, T0, steps, seed = 3, 30, 12, 82
    ca, cb = base, base.with_(is_kv_producer=0)
    wa = synth.layer_weights(ca, seed)
    wb = dict(synth.perturbed_weights(synth.layer_weights(cb, seed + 1), cb, seed + 1), **synth.affine_kv(cb, seed))
    x = synth.layer_input(ca, B, T0 + steps, seed + 2)
    cap = ca.n_meta + ca.window
    g = _Pair(ca, cb, wa, wb, B, T0, cap)
    g.prefill(x[:, :T0])
    o = _oracle_pair(ca, cb, wa, wb, x[:, :T0], cap)
    for t in range(T0, T0 + steps):
        ya, yb = g.step(x[:, t])
        ra = oracle.mixer_decode(ca, wa, x[:, t], o["cache"], o["ha"], o["ca"], residual=True)
        rb = oracle.mixer_decode(cb, wb, ra, o["cache"], o["hb"], o["cb"], residual=True)
        assert_close(to_np(yb), rb, cb, f"consumer step {t}")
    assert g.hy.hymba_get_device_status(None) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_decode_batch(dtype):
    """One decode batch whose sequences sit at different positions (prompts of 5, 13 and
    22 tokens prefilled one by one into their slices of the shared cache and state; the
    8-slot rings at different phases of their wrap): each sequence's outputs match the
    oracle's decode of that sequence, with no padding."""
    torch = torch_cuda()
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt
    if dtype == "f32":
        base = synth.tiny_layer_cfg().with_(window=8)
    else:
        base = synth.hymba15_layer_cfg(window=8).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                       dt_rank=24, n_meta=8)
    ca, cb = base, base.with_(is_kv_producer=0)
    wa = synth.perturbed_weights(synth.layer_weights(ca, 93), ca, 93)
    wb = synth.perturbed_weights(synth.layer_weights(cb, 94), cb, 94)
    lens, steps = (5, 13, 22), 9
    B, m, cap = len(lens), ca.n_meta, ca.n_meta + 8
    x = synth.layer_input(ca, B, max(lens) + steps, 95)
    la, lb = rt.DeviceLayer(ca, wa), rt.DeviceLayer(cb, wb)
    fl = rt.stream_flags(ca)
    io = torch.float32 if (fl & hy.HYMBA_IO_F32 or ca.dtype == 0) else rt.act_dtype(ca)
    kv = rt.KV(ca, B, cache_cap=cap)
    sa, sb = rt.State(ca, B), rt.State(cb, B)
    caches, hs = [], []
    for b, T0 in enumerate(lens):
        # sequence b alone (B = 1) into its slice of the batch's cache and state
        Tp = m + T0
        kseq = torch.empty((1, ca.n_kv_heads, Tp, ca.head_dim), dtype=rt.mid_dtype(ca), device="cuda")
        vseq = torch.empty((1, ca.n_kv_heads, Tp, ca.v_head_dim), dtype=rt.mid_dtype(ca), device="cuda")
        kvs = hy.kv_struct(ca, 1, kseq, vseq, kv.k_cache[b:b + 1], kv.v_cache[b:b + 1], kv.len[b:b + 1])
        kvc = hy.hymba_kv()
        hy.check(hy.hymba_kv_share(ctypes.byref(kvs), ctypes.byref(lb.c), ctypes.byref(kvc)))
        xb = rt.to_device(x[b:b + 1, :T0], ca, io_f32=io == torch.float32)
        ya = torch.empty((1, Tp, ca.d_model), dtype=io, device="cuda")
        yb = torch.empty_like(ya)
        ws = rt.workspace(ca, 1, T0, hy.HYMBA_MODE_PREFILL)
        sta = hy.state_struct(sa.h[b:b + 1], sa.conv[b:b + 1])
        stb = hy.state_struct(sb.h[b:b + 1], sb.conv[b:b + 1])
        hy.check(hy.hymba_mixer_prefill(ctypes.byref(la.c), ctypes.byref(la.s), xb.data_ptr(), 1, T0, fl,
                                        ya.data_ptr(), ctypes.byref(kvs), ctypes.byref(sta), ws.data_ptr(),
                                        ws.numel(), hy.current_stream_ptr()))
        hy.check(hy.hymba_mixer_prefill(ctypes.byref(lb.c), ctypes.byref(lb.s), ya.data_ptr(), 1, T0,
                                        fl | hy.HYMBA_X_HAS_META, yb.data_ptr(), ctypes.byref(kvc),
                                        ctypes.byref(stb), ws.data_ptr(), ws.numel(), hy.current_stream_ptr()))
        pa = oracle.mixer_prefill(ca, wa, x[b:b + 1, :T0], residual=True)
        pb = oracle.mixer_prefill(cb, wb, pa["y"], kv_shared=(pa["k"], pa["v"]), residual=True, x_has_meta=True)
        caches.append(oracle.cache_from_prefill(ca, pa["k"], pa["v"], cap))
        hs.append((pa["h"], pa["conv"], pb["h"], pb["conv"]))
    torch.cuda.synchronize()
    assert kv.len.cpu().tolist() == [m + T0 for T0 in lens]
    cache = {k: np.concatenate([c[k] for c in caches]) for k in ("k", "v", "len")}
    ha, conva, hb, convb = (np.concatenate([h[i] for h in hs]) for i in range(4))
    kvb = hy.hymba_kv()
    hy.check(hy.hymba_kv_share(ctypes.byref(kv.s), ctypes.byref(lb.c), ctypes.byref(kvb)))
    wda = rt.workspace(ca, B, cap, hy.HYMBA_MODE_DECODE)
    wdb = rt.workspace(cb, B, cap, hy.HYMBA_MODE_DECODE)
    for s in range(steps):
        xt_np = np.stack([x[b, lens[b] + s] for b in range(B)])
        xt = rt.to_device(xt_np, ca, io_f32=io == torch.float32)
        ya, yb = torch.empty_like(xt), torch.empty_like(xt)
        rt.decode(la, xt, kv.s, sa, ya, wda, fl)
        rt.decode(lb, ya, kvb, sb, yb, wdb, fl)
        ra = oracle.mixer_decode(ca, wa, xt_np, cache, ha, conva, residual=True)
        rb = oracle.mixer_decode(cb, wb, ra, cache, hb, convb, residual=True)
        assert_close(to_np(yb), rb, cb, f"ragged batch, step {s}")
    assert kv.len.cpu().tolist() == [m + T0 + steps for T0 in lens]
    assert hy.hymba_get_device_status(None) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pair_decode_with_concat_fusion(dtype):
    """Decode through a KV-sharing pair with the concat fusion and 64-wide V heads: the
    decode attention's 64-wide partials, their merge and the wider W_o."""
    if dtype == "f32":
        base = synth.tiny_layer_cfg().with_(window=8, fusion=1, v_head_dim=64)
        B, T0, steps, seed = 2, 10, 10, 121
    else:
        base = synth.hymba15_layer_cfg(window=24).with_(d_model=256, n_q_heads=5, n_kv_heads=1, d_inner=640,
                                                        dt_rank=24, n_meta=8, fusion=1, v_head_dim=64)
        B, T0, steps, seed = 3, 30, 10, 122
    ca, cb = base, base.with_(is_kv_producer=0)
    if dtype == "f32":
        wa = synth.perturbed_weights(synth.layer_weights(ca, seed), ca, seed)
        wb = synth.perturbed_weights(synth.layer_weights(cb, seed + 1), cb, seed + 1)
    else:
        # the workloads' gains and betas (1), as in the average variant's bf16 decode test:
        # the concatenated branches are not halved, and with gains and betas drawn up to
        # about 2.5 the bf16-rounded decode input alone takes the tails past 2e-2
        wa, wb = synth.layer_weights(ca, seed), synth.layer_weights(cb, seed + 1)
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
    assert g.hy.hymba_get_device_status(None) == 0
