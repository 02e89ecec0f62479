"""Pins of the oracle's whole layer: decode-by-decode equals prefill (through the
ring-buffer wrap), cross-layer KV sharing, fusion invariants, and the pages'
printed cache sizes.

Sources: "Hymba Guide", Cross-Layer KV Cache Sharing (a secondary layer reuses the
primary layer's K and V with no new buffer); "Lecture 04", section 1 (the decode
cache gains one K, V per token) and section 8 (kv_cache_gb, ssm_state_gb and their
printed values); "Jamba: Hybrid SSM-Transformer", section 2 and the Worked Example.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_sizes.json")


def _pair(window=8, seed=21):
    base = synth.tiny_layer_cfg().with_(window=window)
    ca = base.with_(is_kv_producer=1)
    cb = base.with_(is_kv_producer=0)
    wa = synth.perturbed_weights(synth.layer_weights(ca, seed), ca, seed)
    wb = synth.perturbed_weights(synth.layer_weights(cb, seed + 1), cb, seed + 1)
    return ca, cb, wa, wb


@pytest.mark.parametrize("window", [8, 0])
def test_decode_by_decode_equals_prefill_pair(window):
    """Prefill T0 tokens then decode the rest one at a time through a KV-sharing
    pair (residual stack) equals prefilling all T tokens. With window 8 the ring
    of 8 slots wraps several times."""
    ca, cb, wa, wb = _pair(window)
    B, T, T0 = 2, 30, 10
    m = ca.n_meta
    x = synth.layer_input(ca, B, T, 31)
    # reference: the whole sequence at once
    ra = oracle.mixer_prefill(ca, wa, x, residual=True)
    rb = oracle.mixer_prefill(cb, wb, ra["y"], kv_shared=(ra["k"], ra["v"]), residual=True, x_has_meta=True)
    # prefill T0, then decode
    pa = oracle.mixer_prefill(ca, wa, x[:, :T0], residual=True)
    pb = oracle.mixer_prefill(cb, wb, pa["y"], kv_shared=(pa["k"], pa["v"]), residual=True, x_has_meta=True)
    cap = m + (window if window > 0 else T)
    cache = oracle.cache_from_prefill(ca, pa["k"], pa["v"], cap)
    ha, conva = pa["h"].copy(), pa["conv"].copy()
    hb, convb = pb["h"].copy(), pb["conv"].copy()
    for t in range(T0, T):
        ya = oracle.mixer_decode(ca, wa, x[:, t], cache, ha, conva, residual=True)
        yb = oracle.mixer_decode(cb, wb, ya, cache, hb, convb, residual=True)
        np.testing.assert_allclose(ya, ra["y"][:, m + t], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(yb, rb["y"][:, m + t], rtol=1e-10, atol=1e-10)
        assert list(cache["len"]) == [m + t + 1] * B
    np.testing.assert_allclose(ha, ra["h"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(hb, rb["h"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(conva, ra["conv"], rtol=0, atol=1e-12)


def test_decode_resumes_from_a_state_snapshot():
    """The decode state is the cache (meta block, ring, len), h and the conv state and
    nothing else: decoding on from a copy of them gives the same outputs, bit for bit,
    as decoding on from the originals."""
    import copy
    ca, cb, wa, wb = _pair(8, seed=41)
    B, T, T0, T1 = 2, 24, 6, 13
    x = synth.layer_input(ca, B, T, 43)
    pa = oracle.mixer_prefill(ca, wa, x[:, :T0], residual=True)
    pb = oracle.mixer_prefill(cb, wb, pa["y"], kv_shared=(pa["k"], pa["v"]), residual=True, x_has_meta=True)
    cache = oracle.cache_from_prefill(ca, pa["k"], pa["v"], ca.n_meta + 8)
    st = [pa["h"].copy(), pa["conv"].copy(), pb["h"].copy(), pb["conv"].copy()]

    def run(cache, st, t0, t1):
        out = []
        for t in range(t0, t1):
            ya = oracle.mixer_decode(ca, wa, x[:, t], cache, st[0], st[1], residual=True)
            out.append(oracle.mixer_decode(cb, wb, ya, cache, st[2], st[3], residual=True))
        return out

    run(cache, st, T0, T1)
    snap_cache, snap_st = copy.deepcopy(cache), [a.copy() for a in st]
    first = run(cache, st, T1, T)
    again = run(snap_cache, snap_st, T1, T)
    for a, b in zip(first, again):
        assert np.array_equal(a, b)
    for a, b in zip(st, snap_st):
        assert np.array_equal(a, b)


def test_ring_slots_closed_form():
    """Meta positions keep slots 0..m-1; position p >= m goes to m + (p - m) mod R."""
    m, R = 3, 4
    got = [oracle.ring_slot(p, m, R) for p in range(13)]
    assert got == [0, 1, 2, 3, 4, 5, 6, 3, 4, 5, 6, 3, 4]
    cfg = synth.tiny_layer_cfg().with_(n_meta=m)
    k = np.arange(13, dtype=np.float64).reshape(1, 1, 13, 1) * np.ones((1, 1, 13, 2))
    c = oracle.cache_from_prefill(cfg, k, k, m + R)
    np.testing.assert_array_equal(c["k"][0, 0, :, 0], [0, 1, 2, 11, 12, 9, 10])


def test_kv_share_consumer_equals_producer_with_same_kv():
    """A consumer reading K, V handed over from a producer (no K/V rows of its own)
    equals the producer itself when the handed-over K, V are the producer's."""
    cfg = synth.tiny_layer_cfg()
    w = synth.perturbed_weights(synth.layer_weights(cfg, 41), cfg, 41)
    x = synth.layer_input(cfg, 1, 20, 41)
    rp = oracle.mixer_prefill(cfg, w, x)
    cc = cfg.with_(is_kv_producer=0)
    H, G, dh, dv, d = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim, cfg.d_model
    wc = dict(w)
    wc["w_in"] = np.concatenate([w["w_in"][:H * dh], w["w_in"][H * dh + G * (dh + dv):]], axis=0)
    assert wc["w_in"].shape[0] == cc.n_in
    rc = oracle.mixer_prefill(cc, wc, x, kv_shared=(rp["k"], rp["v"]))
    np.testing.assert_allclose(rc["y"], rp["y"], rtol=1e-12, atol=1e-12)


def test_rmsnorm_scale_invariance_and_unit_rms():
    g = np.random.default_rng(51)
    a = g.standard_normal((7, 33))
    one = np.ones(33)
    n = oracle.rms_norm(a, one, 0.0)
    np.testing.assert_allclose(oracle.rms_norm(3.7 * a, one, 0.0), n, rtol=1e-13)
    np.testing.assert_allclose(np.sqrt(np.mean(n * n, axis=1)), 1.0, rtol=1e-13)
    gain = g.standard_normal(33)
    np.testing.assert_allclose(oracle.rms_norm(a, gain, 0.0), gain * n, rtol=1e-13)


def test_fuse_beta2_zero_drops_ssm_branch():
    g = np.random.default_rng(52)
    di = 12
    w = {"norm_attn_w": g.standard_normal(di), "norm_ssm_w": g.standard_normal(di),
         "beta1": g.standard_normal(di), "beta2": np.zeros(di)}
    o = g.standard_normal((5, di))
    u1 = oracle.fuse(o, g.standard_normal((5, di)), w, 1e-6)
    u2 = oracle.fuse(o, g.standard_normal((5, di)) * 100.0, w, 1e-6)
    np.testing.assert_array_equal(u1, u2)
    # the average: equal branches with unit gains and betas give RMS(a)
    w1 = {k: np.ones(di) for k in w}
    np.testing.assert_allclose(oracle.fuse(o, o, w1, 0.0), oracle.rms_norm(o, np.ones(di), 0.0), rtol=1e-14)


def test_cache_sizes_match_pages():
    gold = json.load(open(GOLDEN))
    ex = gold["jamba_worked_example"]
    assert oracle.kv_cache_bytes(1, 8, 128, 1, 1, 2) == ex["bytes_per_token_layer"]
    assert oracle.kv_cache_bytes(1, 8, 128, 1, 1, 1) == ex["elements_per_token_layer"]
    assert oracle.kv_cache_bytes(32, 8, 128, 1, 1, 2) == ex["bytes_per_token_32_layers"]
    assert oracle.kv_cache_bytes(32, 8, 128, 64000, 4, 2) == ex["dense_32_layers_bytes"]
    assert oracle.kv_cache_bytes(4, 8, 128, 64000, 4, 2) == ex["hybrid_4_layers_bytes"]
    code = gold["jamba_code_output"]
    t = oracle.kv_cache_bytes(32, 8, 128, code["seq_len"], 1, 2) / 1024 ** 3
    h = oracle.kv_cache_bytes(32 // 8, 8, 128, code["seq_len"], 1, 2) / 1024 ** 3
    assert f"{t:.2f}" == code["transformer_gib_2dp"]
    assert f"{h:.2f}" == code["hybrid_gib_2dp"]
    assert f"{t / h:.1f}" == code["factor_1dp"]
    lec = gold["lecture04_section8"]
    dense70 = oracle.kv_cache_bytes(80, 8, 128, 128_000, 1, 2) / 1e9
    state = oracle.ssm_state_bytes(64, 64 * 64, 128, 1, 2) / 1e9
    dense7 = oracle.kv_cache_bytes(32, 8, 128, 128_000, 1, 2) / 1e9
    assert round(dense70) == lec["dense70b_128k_gb_approx"]
    assert round(state, 2) == lec["ssm_state_gb_approx"]
    assert round(dense7) == lec["dense7b_128k_gb_approx"]
    assert round(dense7 / state, -1) == lec["ratio_approx"]


def test_layer_cache_bytes_formula():
    """KV slots (meta + window) for a producer, fp32 state, conv state, lengths."""
    cfg = synth.hymba15_layer_cfg(1024)
    B = 64
    kv = B * 5 * (128 + 1024) * (64 + 128) * 2
    h = B * 3200 * 16 * 4
    conv = B * 3200 * 4 * 4
    assert oracle.layer_cache_bytes(cfg, B, 4096 + 128) == kv + h + conv + B * 4
    g = cfg.with_(window=0)
    assert oracle.layer_cache_bytes(g, B, 5000) == B * 5 * 5000 * 192 * 2 + h + conv + B * 4


def test_rmsnorm_epsilon_sits_inside_the_square_root():
    """RMS(a) = gain * a / sqrt(mean(a^2) + eps): with mean(a^2) = 1 and eps = 3 the
    divisor is sqrt(4) = 2 exactly, where eps outside the root would give 1 + 3 = 4
    and eps dropped would give 1."""
    a = np.array([[1.0, -1.0, 1.0, -1.0]])
    got = oracle.rms_norm(a, np.ones(4), 3.0)
    np.testing.assert_array_equal(got, a / 2.0)
    # a second closed form: mean(a^2) = 12.5 for a = (3, 4) doubled over 4 columns;
    # eps = 3.5 makes the divisor sqrt(16) = 4
    b = np.array([[3.0, 4.0, -3.0, -4.0]])
    np.testing.assert_array_equal(oracle.rms_norm(b, np.full(4, 2.0), 3.5), 2.0 * b / 4.0)


@pytest.mark.parametrize("window,producer", [(8, 1), (0, 1), (8, 0)])
def test_layer_cache_bytes_counts_the_decode_state_arrays(window, producer):
    """The decode-state size equals the elements of the arrays that one decode step
    reads and writes, counted from the arrays themselves: the cache a prefill leaves
    (producer only; meta slots + ring, or the whole history for a global layer), the
    SSM state h, the conv state and the lengths, at 2 bytes per K/V element for a
    bf16 layer (4 for fp32) and 4 bytes for the fp32 states and int32 lengths."""
    for dtype in (synth.F32, synth.BF16):
        cfg = synth.tiny_layer_cfg().with_(window=window, is_kv_producer=producer, dtype=dtype)
        B, T = 2, 21
        w = synth.layer_weights(cfg, 61)
        x = synth.layer_input(cfg, B, T, 61)
        max_T = cfg.n_meta + T
        kv_src = None
        if not producer:
            p = oracle.mixer_prefill(cfg.with_(is_kv_producer=1), synth.layer_weights(cfg.with_(is_kv_producer=1), 62), x)
            kv_src = (p["k"], p["v"])
        r = oracle.mixer_prefill(cfg, w, x, kv_shared=kv_src)
        cap = cfg.n_meta + (window if window > 0 else T)
        kv_elems = 0
        if producer:
            cache = oracle.cache_from_prefill(cfg, r["k"], r["v"], cap)
            kv_elems = cache["k"].size + cache["v"].size
            assert cache["len"].size == B
        esz = 2 if dtype == synth.BF16 else 4
        counted = kv_elems * esz + r["h"].size * 4 + r["conv"].size * 4 + B * 4
        assert oracle.layer_cache_bytes(cfg, B, max_T) == counted


@pytest.mark.parametrize("window", [8, 0])
def test_decode_equals_prefill_with_affine_shared_kv(window):
    """A consumer that adapts the shared K, V ("Hymba Guide", Cross-Layer KV Cache
    Sharing) decodes as it prefills: the adaptation acts on the cached K, V the same way
    in both paths (the ring of 8 slots wraps several times)."""
    ca, cb, wa, wb = _pair(window, seed=71)
    wb = dict(wb, **synth.affine_kv(cb, 71))
    B, T, T0 = 2, 26, 9
    m = ca.n_meta
    x = synth.layer_input(ca, B, T, 72)
    ra = oracle.mixer_prefill(ca, wa, x, residual=True)
    rb = oracle.mixer_prefill(cb, wb, ra["y"], kv_shared=(ra["k"], ra["v"]), residual=True, x_has_meta=True)
    plain = oracle.mixer_prefill(cb, _pair(window, seed=71)[3], ra["y"], kv_shared=(ra["k"], ra["v"]),
                                 residual=True, x_has_meta=True)
    assert np.abs(rb["y"] - plain["y"]).max() > 1e-3  # the adaptation changes the output
    pa = oracle.mixer_prefill(ca, wa, x[:, :T0], residual=True)
    pb = oracle.mixer_prefill(cb, wb, pa["y"], kv_shared=(pa["k"], pa["v"]), residual=True, x_has_meta=True)
    cap = m + (window if window > 0 else T)
    cache = oracle.cache_from_prefill(ca, pa["k"], pa["v"], cap)
    ha, conva, hb, convb = pa["h"].copy(), pa["conv"].copy(), pb["h"].copy(), pb["conv"].copy()
    for t in range(T0, T):
        ya = oracle.mixer_decode(ca, wa, x[:, t], cache, ha, conva, residual=True)
        yb = oracle.mixer_decode(cb, wb, ya, cache, hb, convb, residual=True)
        np.testing.assert_allclose(yb, rb["y"][:, m + t], rtol=1e-10, atol=1e-10)


def test_ragged_decode_batch_equals_each_sequence_prefilled():
    """Sequences of one decode batch may sit at different positions: each keeps its own
    length, ring slot and state ("51cto" Hymba-1.5B article, section 4, notes that the
    released code wants batch 1 for generation because padded meta tokens and the
    sliding window do not mix; a per-sequence position needs no padding). Three
    sequences prefilled alone with 5, 13 and 22 tokens (window 8: rings at different
    phases of their wrap) and then decoded together equal each sequence prefilled at
    its final length."""
    ca, cb, wa, wb = _pair(8, seed=91)
    m, cap = ca.n_meta, ca.n_meta + 8
    lens, steps = (5, 13, 22), 9
    B = len(lens)
    x = synth.layer_input(ca, B, max(lens) + steps, 92)
    caches, hs = [], []
    for b, T0 in enumerate(lens):
        pa = oracle.mixer_prefill(ca, wa, x[b:b + 1, :T0], residual=True)
        pb = oracle.mixer_prefill(cb, wb, pa["y"], kv_shared=(pa["k"], pa["v"]), residual=True, x_has_meta=True)
        caches.append(oracle.cache_from_prefill(ca, pa["k"], pa["v"], cap))
        hs.append((pa["h"], pa["conv"], pb["h"], pb["conv"]))
    cache = {k: np.concatenate([c[k] for c in caches]) for k in ("k", "v", "len")}
    ha, conva, hb, convb = (np.concatenate([h[i] for h in hs]) for i in range(4))
    for s in range(steps):
        xt = np.stack([x[b, lens[b] + s] for b in range(B)])
        ya = oracle.mixer_decode(ca, wa, xt, cache, ha, conva, residual=True)
        yb = oracle.mixer_decode(cb, wb, ya, cache, hb, convb, residual=True)
        for b, T0 in enumerate(lens):
            ra = oracle.mixer_prefill(ca, wa, x[b:b + 1, :T0 + s + 1], residual=True)
            rb = oracle.mixer_prefill(cb, wb, ra["y"], kv_shared=(ra["k"], ra["v"]), residual=True, x_has_meta=True)
            np.testing.assert_allclose(yb[b], rb["y"][0, -1], rtol=1e-10, atol=1e-10)
    assert list(cache["len"]) == [m + T0 + steps for T0 in lens]


def _concat_cfg():
    """The tiny layer with the concat fusion ("Hymba Guide", Parallel Hybrid-Head Layer
    Formulation: y = W_o(Concat[MambaHeads(x), AttentionHeads(x)])), V head dim = 64."""
    return synth.tiny_layer_cfg().with_(fusion=1, v_head_dim=64)


def test_concat_fusion_is_the_sum_of_the_two_partial_products():
    """W_o applied to [Mamba | Attention] equals W_o's first d_inner columns applied to
    the normalised Mamba branch plus its last H * dv columns applied to the normalised
    attention branch; widths d_inner + H * dv."""
    cfg = _concat_cfg()
    w = synth.perturbed_weights(synth.layer_weights(cfg, 101), cfg, 101)
    x = synth.layer_input(cfg, 1, 30, 101)
    r = oracle.mixer_prefill(cfg, w, x)
    di, hv = cfg.d_inner, cfg.n_q_heads * cfg.v_head_dim
    assert r["u"].shape[-1] == di + hv == w["w_out"].shape[1]
    s = oracle.rms_norm(r["y_ssm"], w["norm_ssm_w"].astype(np.float64), cfg.rms_eps) * w["beta2"]
    a = oracle.rms_norm(r["o_attn"], w["norm_attn_w"].astype(np.float64), cfg.rms_eps) * w["beta1"]
    wo = w["w_out"].astype(np.float64)
    np.testing.assert_allclose(r["y"], s @ wo[:, :di].T + a @ wo[:, di:].T, rtol=1e-10, atol=1e-12)


def test_concat_with_equal_halves_is_twice_the_average():
    """With equal branch widths and W_o = [W | W], the concatenation gives 2 * the
    beta-average through W: both fusions share the per-branch norm and beta scaling."""
    base = synth.tiny_layer_cfg()
    cat = base.with_(fusion=1)  # v_head_dim 128: H * dv = d_inner
    w = synth.perturbed_weights(synth.layer_weights(base, 102), base, 102)
    wc = dict(w, w_out=np.concatenate([w["w_out"], w["w_out"]], axis=1))
    x = synth.layer_input(base, 1, 25, 102)
    ra = oracle.mixer_prefill(base, w, x)
    rc = oracle.mixer_prefill(cat, wc, x)
    np.testing.assert_allclose(rc["y"], 2.0 * ra["y"], rtol=1e-10, atol=1e-12)


def test_concat_beta1_zero_drops_attention():
    cfg = _concat_cfg()
    w = synth.layer_weights(cfg, 103)
    w = dict(w, beta1=np.zeros_like(w["beta1"]))
    x = synth.layer_input(cfg, 1, 20, 103)
    r = oracle.mixer_prefill(cfg, w, x)
    assert np.all(r["u"][..., cfg.d_inner:] == 0.0)


# ---------------------------------------------------------------------------
# the block around the mixer: pre-norm residual mixer, pre-norm SiLU-gated MLP
# ("51cto" Hymba-1.5B article, section 2: MLP intermediate size 5504)
# ---------------------------------------------------------------------------

def test_mlp_hand_worked():
    """d = 2, d_ff = 1: n = RMSNorm(h) = h / rms(h) = (1, 1) for h = (3, 3); gate row
    (ln 3, 0) gives SiLU(ln 3) = ln 3 * 3/4; up row (2, 0) gives 2; down column (1, -1)."""
    h = np.array([[3.0, 3.0]])
    w = {"norm_w": np.ones(2), "w_gate": np.array([[np.log(3.0), 0.0]]), "w_up": np.array([[2.0, 0.0]]),
         "w_down": np.array([[1.0], [-1.0]])}
    a = np.log(3.0) * 0.75 * 2.0
    np.testing.assert_allclose(oracle.mlp(h, w, 0.0), [[3.0 + a, 3.0 - a]], rtol=1e-14)


def test_mlp_zero_down_is_identity_and_scale_invariant_branch():
    g = np.random.default_rng(111)
    w = synth.mlp_weights(32, 48, synth.F32, 111)
    h = g.standard_normal((5, 32))
    np.testing.assert_array_equal(oracle.mlp(h, dict(w, w_down=np.zeros_like(w["w_down"])), 1e-6), h)
    # the branch sees RMSNorm(h): scaling h scales only the residual part
    branch = oracle.mlp(h, w, 0.0) - h
    np.testing.assert_allclose(oracle.mlp(7.0 * h, w, 0.0) - 7.0 * h, branch, rtol=1e-12, atol=1e-12)


def test_block_is_two_pre_norm_residual_steps():
    """block(h) = MLP(h + mixer(RMSNorm(h) g)); with W_out = 0 and W_down = 0 it is the
    identity, and the mixer inside sees the normalised stream (scaling h leaves the
    mixer's output unchanged)."""
    cfg = synth.tiny_layer_cfg().with_(rms_eps=0.0)  # exact scale invariance of the norms
    wm = synth.with_pre_norm(synth.layer_weights(cfg, 112), cfg, 112, scale=0.3)
    wf = synth.mlp_weights(cfg.d_model, 96, cfg.dtype, 113)
    g = np.random.default_rng(114)
    h = g.standard_normal((1, cfg.n_meta + 20, cfg.d_model))
    r = oracle.block_prefill(cfg, wm, wf, h)
    np.testing.assert_allclose(r["y"][0], oracle.mlp(r["h1"][0], wf, cfg.rms_eps), rtol=1e-12)
    zero = oracle.block_prefill(cfg, dict(wm, w_out=np.zeros_like(wm["w_out"])),
                                dict(wf, w_down=np.zeros_like(wf["w_down"])), h)
    np.testing.assert_array_equal(zero["y"], h)
    r3 = oracle.block_prefill(cfg, wm, wf, 3.0 * h)
    np.testing.assert_allclose(r3["h1"] - 3.0 * h, r["h1"] - h, rtol=1e-9, atol=1e-9)


def test_block_decode_equals_block_prefill():
    """A KV-sharing pair of blocks decodes as it prefills (window 8 ring wrapping)."""
    ca, cb, wa, wb = _pair(8, seed=115)
    wa, wb = synth.with_pre_norm(wa, ca, 115, 0.3), synth.with_pre_norm(wb, cb, 116, 0.3)
    fa, fb = synth.mlp_weights(ca.d_model, 64, ca.dtype, 117), synth.mlp_weights(cb.d_model, 64, cb.dtype, 118)
    B, T, T0 = 2, 22, 9
    m = ca.n_meta
    g = np.random.default_rng(119)
    h = g.standard_normal((B, m + T, ca.d_model))
    ra = oracle.block_prefill(ca, wa, fa, h)
    rb = oracle.block_prefill(cb, wb, fb, ra["y"], kv_shared=(ra["k"], ra["v"]))
    pa = oracle.block_prefill(ca, wa, fa, h[:, :m + T0])
    pb = oracle.block_prefill(cb, wb, fb, pa["y"], kv_shared=(pa["k"], pa["v"]))
    cache = oracle.cache_from_prefill(ca, pa["k"], pa["v"], m + 8)
    ha, conva, hb, convb = pa["h"].copy(), pa["conv"].copy(), pb["h"].copy(), pb["conv"].copy()
    for t in range(T0, T):
        ya = oracle.block_decode(ca, wa, fa, h[:, m + t], cache, ha, conva)
        yb = oracle.block_decode(cb, wb, fb, ya, cache, hb, convb)
        np.testing.assert_allclose(yb, rb["y"][:, m + t], rtol=1e-10, atol=1e-10)


def test_decode_after_a_prefill_shorter_than_the_conv():
    """A prefill of fewer rows than the conv width (no meta rows, 2 tokens) leaves a conv
    state whose missing history is zero, so decoding on from it equals prefilling the
    whole sequence (the zero history before the first row of the prefill)."""
    cfg = synth.tiny_layer_cfg().with_(n_meta=0, window=8)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 41), cfg, 41)
    B, T, T0 = 2, 9, 2
    x = synth.layer_input(cfg, B, T, 42)
    ref = oracle.mixer_prefill(cfg, w, x, residual=True)
    pre = oracle.mixer_prefill(cfg, w, x[:, :T0], residual=True)
    assert pre["conv"].shape == (B, cfg.d_inner, cfg.d_conv)
    np.testing.assert_array_equal(pre["conv"][:, :, :cfg.d_conv - T0], 0.0)
    cache = oracle.cache_from_prefill(cfg, pre["k"], pre["v"], cfg.window)
    h, conv = pre["h"].copy(), pre["conv"].copy()
    for t in range(T0, T):
        y = oracle.mixer_decode(cfg, w, x[:, t], cache, h, conv, residual=True)
        np.testing.assert_allclose(y, ref["y"][:, t], rtol=1e-10, atol=1e-10)
